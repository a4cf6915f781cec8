// probe.cu -- a measurement aid: the FP32 SIMT lane-operation rate of the device.
//
// The roofline of the LNQ codebook and assignment steps counts FP32 lane operations (one FADD or
// FFMA by one lane). Its denominator is measured with this kernel rather than derived from the
// data sheet: every thread runs eight independent FFMA chains, enough warps are resident to hide
// the FFMA latency, and the caller times the launch with CUDA events.
#include "common.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kProbeThreads = 256;
constexpr int kProbeBlocksPerSm = 8;  // 2048 threads: every warp slot of an SM
constexpr int kProbeChains = 8;

__global__ void __launch_bounds__(kProbeThreads)
    fp32_probe_kernel(int64_t iters, float *__restrict__ sink)
{
    float a[kProbeChains];
#pragma unroll
    for (int c = 0; c < kProbeChains; ++c)
        a[c] = static_cast<float>(threadIdx.x + c);
    const float b = 0.999999f, k = 1e-6f;  // each chain converges to k / (1 - b), stays finite
    for (int64_t it = 0; it < iters; it += 16) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
#pragma unroll
            for (int c = 0; c < kProbeChains; ++c)
                a[c] = fmaf(a[c], b, k);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kProbeChains; ++c)
        s += a[c];
    if (s == -1.f)  // never true; keeps the chains live
        sink[0] = s;
}

}  // namespace lnq

extern "C" LNQ_API lnq_status lnq_fp32_probe(int64_t iters, float *sink, int64_t *lane_ops,
                                             lnq_stream_t stream)
{
    if (iters < 16 || iters % 16 != 0 || sink == nullptr || lane_ops == nullptr)
        return LNQ_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        return LNQ_ERR_CUDA;
    const unsigned blocks = static_cast<unsigned>(sms * lnq::kProbeBlocksPerSm);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    {
        lnq::KernelTimer timer("fp32_probe", s);
        lnq::fp32_probe_kernel<<<blocks, lnq::kProbeThreads, 0, s>>>(iters, sink);
    }
    if (cudaGetLastError() != cudaSuccess)
        return LNQ_ERR_CUDA;
    *lane_ops = static_cast<int64_t>(blocks) * lnq::kProbeThreads * iters * lnq::kProbeChains;
    return LNQ_OK;
}
