// noalloc.cu -- lnq_build_fisher_noalloc: the guided Fisher build without a caller-provided
// workspace.
//
// Some callers cannot allocate device memory at the moment they want F. Examples: code that
// runs inside another framework's fixed memory pool, or a plugin with no allocator handle. Code
// on a latency-critical path cannot afford the implicit synchronisation of cudaMalloc either.
// For them the scratch this computation needs lives in a file-scope device array that is part of
// the library image: every GPU that loads the library holds these LNQ_NOALLOC_SCRATCH_BYTES until
// the process exits.
//
// The array's name in host code is only a host-side stand-in, not a device address. Its device
// address is looked up once per device with cudaGetSymbolAddress (with that device current) and
// then passed to the kernels.
#include <mutex>

#include "common.cuh"
#include "lnq_internal.cuh"

namespace lnq {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LNQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void *g_addr[kMaxDevices] = {};

}  // namespace

// Device address of the scratch array on the current device; nullptr if it cannot be found.
// Looked up once per device and cached: the cached address does not survive a cudaDeviceReset of
// that device (the library must not be used across one).
void *noalloc_scratch_address()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lk(g_addr_mu);
    if (g_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess)
            return nullptr;
        g_addr[dev] = p;
    }
    return g_addr[dev];
}

}  // namespace lnq

extern "C" LNQ_API lnq_status lnq_build_fisher_noalloc(const uint16_t *X, const uint16_t *G,
                                                       int64_t n, int64_t d_in, int64_t d_out,
                                                       int groups, float alpha, float *F,
                                                       lnq_stream_t stream)
{
    // Reject problems that need more scratch than the static array holds, before touching the
    // device. Invalid sizes (need == 0) fall through to the argument checks of lnq_build_fisher.
    const size_t need = (G == nullptr)
                            ? lnq::kWsHeader
                            : lnq_workspace_size(LNQ_OP_BUILD_FISHER, n, d_in, d_out, groups, 0);
    if (need > static_cast<size_t>(LNQ_NOALLOC_SCRATCH_BYTES))
        return LNQ_ERR_WORKSPACE;
    void *scratch = lnq::noalloc_scratch_address();
    if (scratch == nullptr)
        return LNQ_ERR_CUDA;
    // The regular entry point zeroes what must start at zero (the error header and the per-group
    // maxima) on `stream` before any kernel reads it, and overwrites everything else.
    return lnq_build_fisher(X, G, n, d_in, d_out, groups, alpha, F, scratch,
                            static_cast<size_t>(LNQ_NOALLOC_SCRATCH_BYTES), stream);
}
