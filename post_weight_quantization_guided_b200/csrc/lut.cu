// lut.cu -- the consumer of (C, Q): packed low-bit codes and the lookup-table GEMV on sm_100a.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section, last sentence (LNQ runs on the same
// CUDA kernel as SqueezeLLM), and the aitopics "squeezellm" tag page: the SqueezeLLM abstract
// (single-batch generation is bound by memory bandwidth, so weights are kept as low-bit indices)
// and the GANQ abstract (lookup-table based mixed-precision GEMM). y = x W^T with W^[j][i] =
// c_j[q_ji]: the weights stay packed in HBM and are read once, through each row's codebook.
//
// Packed format (the pages fix none): bits = log2(m); a row is a run of 32-bit words holding
// floor(32 / bits) codes each (8 at 4 bits, 10 at 3 bits, 16 at 2 bits, 32 at 1 bit), code i of
// the row in word i / floor(32 / bits) at bit (i mod floor(32 / bits)) * bits; unused bits are
// zero. No code straddles two words, so a word decodes on its own.
//
// Kernels:
//   pack_codes_kernel  one thread per output word: reads its codes, writes the word.
//   lut_gemv_kernel    one warp per output row: the row's codebook in shared memory, lane l takes
//                      words l, l + 32, ... (coalesced; 8 loads in flight per lane before any is
//                      decoded), decodes each code once and multiplies it
//                      with the NB (1..8, a template parameter) activation vectors (read through the read-only cache; they
//                      are shared by every row), fp32 sums per lane, then a fixed-order warp tree.
//                      Bound: HBM, the packed codes read once (d_out * words * 4 bytes).
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kLutWarps = 8;      // rows per CTA
constexpr int kLutUnroll = 8;     // words a lane has in flight before decoding them

__host__ __device__ inline int64_t lut_words(int64_t d_in, int bits)
{
    const int64_t per = 32 / bits;
    return (d_in + per - 1) / per;
}

__global__ void __launch_bounds__(256)
    pack_codes_kernel(const uint8_t *__restrict__ Q, int64_t d_out, int64_t d_in, int bits,
                      uint32_t *__restrict__ P)
{
    const int per = 32 / bits;
    const int64_t words = lut_words(d_in, bits);
    const int64_t total = d_out * words;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = e / words, w = e - j * words;
        const int64_t i0 = w * per;
        const int n = static_cast<int>(min(static_cast<int64_t>(per), d_in - i0));
        const uint8_t *q = Q + j * d_in + i0;
        uint32_t word = 0u;
        for (int t = 0; t < n; ++t)
            word |= (static_cast<uint32_t>(q[t]) & mask) << (t * bits);
        P[e] = word;
    }
}

template <int BITS, int NB>
__global__ void __launch_bounds__(kLutWarps * 32)
    lut_gemv_kernel(const float *__restrict__ x, const uint32_t *__restrict__ P,
                    const float *__restrict__ C, int64_t d_out, int64_t d_in,
                    float *__restrict__ y)
{
    constexpr int PER = 32 / BITS;
    constexpr int M = 1 << BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    __shared__ float cs[kLutWarps][M];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t words = lut_words(d_in, BITS);
    const bool vec = (PER % 4 == 0) && (d_in % 4 == 0) && (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * kLutWarps + warp; j < d_out;
         j += static_cast<int64_t>(gridDim.x) * kLutWarps) {
        if (lane < M)
            cs[warp][lane] = C[j * M + lane];
        __syncwarp();
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b)
            acc[b] = 0.f;
        const uint32_t *pj = P + j * words;
        for (int64_t w0 = lane; w0 < words; w0 += 32 * kLutUnroll) {
          // the lane's next kLutUnroll words, all loads issued before the first is used
          uint32_t wd[kLutUnroll];
#pragma unroll
          for (int u = 0; u < kLutUnroll; ++u) {
            const int64_t w = w0 + 32 * u;
            wd[u] = w < words ? __ldg(pj + w) : 0u;
          }
#pragma unroll
          for (int u = 0; u < kLutUnroll; ++u) {
            const int64_t w = w0 + 32 * u;
            if (w >= words)
                continue;
            const uint32_t word = wd[u];
            const int64_t i0 = w * PER;
            float wv[PER];
#pragma unroll
            for (int t = 0; t < PER; ++t)
                wv[t] = cs[warp][(word >> (t * BITS)) & MASK];
            if (vec && i0 + PER <= d_in) {
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const float4 *xb = reinterpret_cast<const float4 *>(x + b * d_in + i0);
#pragma unroll
                    for (int t4 = 0; t4 < PER / 4; ++t4) {
                        const float4 v = __ldg(xb + t4);
                        acc[b] = fmaf(v.x, wv[4 * t4], acc[b]);
                        acc[b] = fmaf(v.y, wv[4 * t4 + 1], acc[b]);
                        acc[b] = fmaf(v.z, wv[4 * t4 + 2], acc[b]);
                        acc[b] = fmaf(v.w, wv[4 * t4 + 3], acc[b]);
                    }
                }
            } else {
#pragma unroll
                for (int b = 0; b < NB; ++b) {
#pragma unroll
                    for (int t = 0; t < PER; ++t)
                        if (i0 + t < d_in)
                            acc[b] = fmaf(__ldg(x + b * d_in + i0 + t), wv[t], acc[b]);
                }
            }
          }
        }
        // fixed-order warp tree
#pragma unroll
        for (int b = 0; b < NB; ++b) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
                y[b * d_out + j] = acc[b];
        }
        __syncwarp();  // the row's codebook is read before the next row overwrites it
    }
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
int64_t lnq_lut_words(int64_t d_in, int bits) { return lut_words(d_in, bits); }

cudaError_t lnq_pack_launch(const uint8_t *Q, int64_t d_out, int64_t d_in, int bits, uint32_t *P,
                            int num_sms, cudaStream_t s)
{
    const int64_t total = d_out * lut_words(d_in, bits);
    int64_t blocks = (total + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 32)
        blocks = static_cast<int64_t>(num_sms) * 32;
    KernelTimer timer("lnq_pack_codes", s);
    pack_codes_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(Q, d_out, d_in, bits, P);
    return cudaGetLastError();
}

template <int BITS, int NB>
static cudaError_t lut_gemv_nb(const float *x, const uint32_t *P, const float *C, int64_t d_out,
                               int64_t d_in, float *y, int num_sms, cudaStream_t s)
{
    int64_t blocks = (d_out + kLutWarps - 1) / kLutWarps;
    if (blocks > static_cast<int64_t>(num_sms) * 16)
        blocks = static_cast<int64_t>(num_sms) * 16;
    KernelTimer timer("lnq_lut_gemv", s);
    lut_gemv_kernel<BITS, NB><<<static_cast<unsigned>(blocks), kLutWarps * 32, 0, s>>>(
        x, P, C, d_out, d_in, y);
    return cudaGetLastError();
}

template <int BITS>
static cudaError_t lut_gemv_bits(const float *x, int nb, const uint32_t *P, const float *C,
                                 int64_t d_out, int64_t d_in, float *y, int num_sms, cudaStream_t s)
{
    switch (nb) {
    case 1: return lut_gemv_nb<BITS, 1>(x, P, C, d_out, d_in, y, num_sms, s);
    case 2: return lut_gemv_nb<BITS, 2>(x, P, C, d_out, d_in, y, num_sms, s);
    case 3: return lut_gemv_nb<BITS, 3>(x, P, C, d_out, d_in, y, num_sms, s);
    case 4: return lut_gemv_nb<BITS, 4>(x, P, C, d_out, d_in, y, num_sms, s);
    case 5: return lut_gemv_nb<BITS, 5>(x, P, C, d_out, d_in, y, num_sms, s);
    case 6: return lut_gemv_nb<BITS, 6>(x, P, C, d_out, d_in, y, num_sms, s);
    case 7: return lut_gemv_nb<BITS, 7>(x, P, C, d_out, d_in, y, num_sms, s);
    case 8: return lut_gemv_nb<BITS, 8>(x, P, C, d_out, d_in, y, num_sms, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t lnq_lut_gemv_launch(const float *x, int nb, const uint32_t *P, const float *C,
                                int64_t d_out, int64_t d_in, int bits, float *y, int num_sms,
                                cudaStream_t s)
{
    switch (bits) {
    case 1: return lut_gemv_bits<1>(x, nb, P, C, d_out, d_in, y, num_sms, s);
    case 2: return lut_gemv_bits<2>(x, nb, P, C, d_out, d_in, y, num_sms, s);
    case 3: return lut_gemv_bits<3>(x, nb, P, C, d_out, d_in, y, num_sms, s);
    case 4: return lut_gemv_bits<4>(x, nb, P, C, d_out, d_in, y, num_sms, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
