// profile.cuh -- scoped CUDA-event timer around one kernel launch (active only when profiling
// has been switched on with lnq_profile_enable).
#pragma once

#include <cuda_runtime.h>

#include "../../include/lnq.h"

namespace lnq {

class KernelTimer {
public:
    KernelTimer(const char *name, cudaStream_t s);
    ~KernelTimer();
    KernelTimer(const KernelTimer &) = delete;
    KernelTimer &operator=(const KernelTimer &) = delete;

private:
    const char *name_;
    cudaStream_t stream_;
    cudaEvent_t start_ = nullptr, stop_ = nullptr;
    bool active_ = false;
};

}  // namespace lnq
