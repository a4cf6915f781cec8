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
//   lut_gemv_kernel    K split over the 16 warps of a CTA: lane l of warp w takes the words
//                      w * 32 + l + 512 s of every row, so one set of its activation values serves
//                      every row. A CTA takes R rows at a time (R = 32 / NB, rounded down to a
//                      power of two): their codebooks in shared memory, the R packed words of each
//                      of its slices loaded before any is decoded (R loads in flight per lane),
//                      each code decoded once and multiplied with the NB activation vectors, code
//                      position by code position so that the R rows' sums are independent chains.
//                      Per row a lane sums its words in order; the 32 lanes' sums of the R rows are
//                      reduced by a transposing butterfly of shuffles (lane l ends with row
//                      l / (32 / R)), and the 16 warps' sums are added in order.
//                      Bound: HBM, the packed codes read once (d_out * words * 4 bytes); in
//                      practice the issue rate (about 7 instructions per code: decode, address,
//                      lookup, product, and the loop and reduction around them).
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kLutWarps = 16;                  // K split: warps of a CTA
constexpr int kLutThreads = kLutWarps * 32;

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

// v[r] of every lane summed over the 32 lanes: a butterfly that halves the vector at each step,
// so that lane l ends with the sum for row l / (32 / R). Fixed order, so bit-identical runs.
template <int R>
__device__ __forceinline__ float lut_transpose_sum(float (&v)[R], int lane)
{
#pragma unroll
    for (int n = R / 2, o = 16; n >= 1; n >>= 1, o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int c = 0; c < n; ++c) {
            const float send = upper ? v[c] : v[c + n];
            const float keep = upper ? v[c + n] : v[c];
            v[c] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int o = 16 / R; o >= 1; o >>= 1)
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    return v[0];
}

template <int BITS, int NB, int R>
__global__ void __launch_bounds__(kLutThreads, 1)
    lut_gemv_kernel(const float *__restrict__ x, const uint32_t *__restrict__ P,
                    const float *__restrict__ C, int64_t d_out, int64_t d_in,
                    float *__restrict__ y)
{
    constexpr int PER = 32 / BITS;
    constexpr int M = 1 << BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    static_assert(R >= 1 && R <= 32 && (R & (R - 1)) == 0, "rows per block: a power of two");
    __shared__ float cs[R][M];
    __shared__ float part[NB][kLutWarps][R];
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int64_t words = lut_words(d_in, BITS);
    const int64_t nslice = (words + kLutThreads - 1) / kLutThreads;
    for (int64_t j0 = static_cast<int64_t>(blockIdx.x) * R; j0 < d_out;
         j0 += static_cast<int64_t>(gridDim.x) * R) {
        __syncthreads();   // the previous rows' codebooks and partial sums are read
        for (int e = t; e < R * M; e += kLutThreads) {
            const int64_t j = j0 + e / M;
            cs[e / M][e % M] = j < d_out ? C[j * M + e % M] : 0.f;
        }
        __syncthreads();
        float acc[NB][R];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int r = 0; r < R; ++r)
                acc[b][r] = 0.f;
        for (int64_t s = 0; s < nslice; ++s) {
            const int64_t w = s * kLutThreads + warp * 32 + lane;
            const bool win = w < words;
            uint32_t wd[R];
#pragma unroll
            for (int r = 0; r < R; ++r)
                wd[r] = (win && j0 + r < d_out) ? __ldg(P + (j0 + r) * words + w) : 0u;
#pragma unroll
            for (int tt = 0; tt < PER; ++tt) {
                const int64_t i = w * PER + tt;
                float xv[NB];
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    xv[b] = (win && i < d_in) ? __ldg(x + b * d_in + i) : 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float v = cs[r][(wd[r] >> (tt * BITS)) & MASK];
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        acc[b][r] = fmaf(v, xv[b], acc[b][r]);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const float sum = lut_transpose_sum<R>(acc[b], lane);
            if ((lane & (32 / R - 1)) == 0)
                part[b][warp][lane / (32 / R)] = sum;
        }
        __syncthreads();
        for (int e = t; e < NB * R; e += kLutThreads) {
            const int b = e / R, r = e % R;
            if (j0 + r < d_out) {
                float sum = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kLutWarps; ++w2)
                    sum += part[b][w2][r];
                y[b * d_out + j0 + r] = sum;
            }
        }
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
    // rows per block: 32 / NB rounded down to a power of two (NB * R <= 32 accumulators)
    constexpr int R = NB == 1 ? 32 : (NB == 2 ? 16 : (NB <= 4 ? 8 : 4));
    int64_t blocks = (d_out + R - 1) / R;
    if (blocks > static_cast<int64_t>(num_sms))
        blocks = static_cast<int64_t>(num_sms);
    KernelTimer timer("lnq_lut_gemv", s);
    lut_gemv_kernel<BITS, NB, R><<<static_cast<unsigned>(blocks), kLutThreads, 0, s>>>(
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
