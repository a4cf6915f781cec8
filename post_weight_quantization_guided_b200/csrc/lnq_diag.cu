// lnq_diag.cu -- LNQ with a diagonal Fisher block (the SqueezeLLM-style objective) on sm_100a.
//
// Source: "GuidedQuant" (jinukkim.me blog), opening list, item 2 (diagonal-Fisher methods weight
// the errors by end-loss gradients but keep only the diagonal of the Fisher block), the aitopics
// "squeezellm" tag page, SqueezeLLM abstract (sensitivity-based non-uniform quantization), and
// the blog's LNQ section iteration, applied to F = diag(f). With a diagonal
// block the iteration separates by coordinate:
//   codebook    c_a = sum_{i: q_i = a} f_i w_i / sum_{i: q_i = a} f_i   (the normal equations
//               P^T diag(f) P c = P^T diag(f) w are diagonal), over non-empty codewords; a class
//               whose weights f_i are all 0 is a zero pivot: the row keeps its codebook and is
//               flagged singular, as in the full solve;
//   assignment  moving coordinate i from c_q to c_a changes the objective by
//               f_i ((c_a - w_i)^2 - (c_q - w_i)^2) and changes no other coordinate's term, so
//               every coordinate takes its best codeword at once (lowest index among equals,
//               only a strictly negative change moves).
// diag_lnq_kernel: one CTA per row, the row's weights and codes in shared memory for all
// iterations; class sums in fp64, reduced in a fixed order; the changes in fp64; the objective
// sum_i f_i r_i^2 in fp64.
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kDiagThreads = 256;

template <int M>
__global__ void __launch_bounds__(kDiagThreads)
    diag_lnq_kernel(const float *__restrict__ Fd, const float *__restrict__ W, int64_t d,
                    int64_t rows_per_group, int iters, float *__restrict__ C,
                    uint8_t *__restrict__ Q, double *__restrict__ J, int32_t *__restrict__ status)
{
    extern __shared__ uint8_t dsm[];
    float *ws = reinterpret_cast<float *>(dsm);                          // [d]
    uint8_t *qs = dsm + static_cast<size_t>(d) * 4;                      // [d]
    __shared__ double red[kDiagThreads / 32][2 * M];
    __shared__ double tot[2 * M];
    __shared__ float cb[M];
    __shared__ int flag;
    const int64_t j = blockIdx.x;
    const float *f = Fd + (j / rows_per_group) * d;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    for (int64_t i = t; i < d; i += kDiagThreads) {
        ws[i] = W[j * d + i];
        qs[i] = Q[j * d + i] & (M - 1);
    }
    if (t < M)
        cb[t] = C[j * M + t];
    if (t == 0)
        flag = 0;
    __syncthreads();
    for (int it = 0; it < iters; ++it) {
        // codebook: per class, sum f_i w_i and sum f_i (and whether the class is non-empty)
        double sw[M], sf[M];
        int cnt[M];
#pragma unroll
        for (int a = 0; a < M; ++a) {
            sw[a] = 0.0;
            sf[a] = 0.0;
            cnt[a] = 0;
        }
        for (int64_t i = t; i < d; i += kDiagThreads) {
            const int q = qs[i];
            const double fi = f[i];
#pragma unroll
            for (int a = 0; a < M; ++a) {
                if (q == a) {
                    sw[a] += fi * static_cast<double>(ws[i]);
                    sf[a] += fi;
                    cnt[a] += 1;
                }
            }
        }
        // fixed-order reduction: warp trees, then warps in order
#pragma unroll
        for (int a = 0; a < M; ++a) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sw[a] += __shfl_xor_sync(0xffffffffu, sw[a], o);
                sf[a] += __shfl_xor_sync(0xffffffffu, sf[a], o);
                cnt[a] += __shfl_xor_sync(0xffffffffu, cnt[a], o);
            }
        }
        __shared__ int cntw[kDiagThreads / 32][M];
        if (lane == 0) {
#pragma unroll
            for (int a = 0; a < M; ++a) {
                red[warp][a] = sw[a];
                red[warp][M + a] = sf[a];
                cntw[warp][a] = cnt[a];
            }
        }
        __syncthreads();
        if (t < 2 * M) {
            double s = 0.0;
            for (int w = 0; w < kDiagThreads / 32; ++w)
                s += red[w][t];
            tot[t] = s;
        }
        __syncthreads();
        if (t == 0) {
            bool singular = false;
            for (int a = 0; a < M; ++a) {
                int n = 0;
                for (int w = 0; w < kDiagThreads / 32; ++w)
                    n += cntw[w][a];
                if (n > 0 && !(tot[M + a] > 0.0))
                    singular = true;
            }
            if (singular) {
                flag = 1;
            } else {
                for (int a = 0; a < M; ++a) {
                    int n = 0;
                    for (int w = 0; w < kDiagThreads / 32; ++w)
                        n += cntw[w][a];
                    if (n > 0)
                        cb[a] = static_cast<float>(tot[a] / tot[M + a]);
                }
            }
        }
        __syncthreads();
        // assignment: every coordinate at once (the changes do not interact)
        for (int64_t i = t; i < d; i += kDiagThreads) {
            const double fi = f[i];
            const double wi = ws[i];
            const int q = qs[i];
            const double cur = cb[q];
            double best = 0.0;
            int ba = q;
#pragma unroll
            for (int a = 0; a < M; ++a) {
                const double ca = cb[a];
                const double delta = fi * ((ca - wi) * (ca - wi) - (cur - wi) * (cur - wi));
                if (delta < best) {
                    best = delta;
                    ba = a;
                }
            }
            qs[i] = static_cast<uint8_t>(ba);
        }
        __syncthreads();
    }
    // results: codebook, codes, objective sum_i f_i (c[q_i] - w_i)^2
    if (t < M)
        C[j * M + t] = cb[t];
    double jr = 0.0;
    for (int64_t i = t; i < d; i += kDiagThreads) {
        Q[j * d + i] = qs[i];
        const double r = static_cast<double>(cb[qs[i]]) - static_cast<double>(ws[i]);
        jr += static_cast<double>(f[i]) * r * r;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        jr += __shfl_xor_sync(0xffffffffu, jr, o);
    if (lane == 0)
        red[warp][0] = jr;
    __syncthreads();
    if (t == 0) {
        double s = 0.0;
        for (int w = 0; w < kDiagThreads / 32; ++w)
            s += red[w][0];
        if (J != nullptr)
            J[j] = s;
        if (status != nullptr)
            status[j] = flag ? LNQ_ROW_SINGULAR : LNQ_ROW_OK;
    }
}

template <int M>
static cudaError_t diag_m(const float *Fd, const float *W, int64_t d_out, int64_t d,
                          int64_t rows_per_group, int iters, float *C, uint8_t *Q, double *J,
                          int32_t *status, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>(d) * 5;
    cudaError_t e = cudaFuncSetAttribute(diag_lnq_kernel<M>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    KernelTimer timer("lnq_diag", s);
    diag_lnq_kernel<M><<<static_cast<unsigned>(d_out), kDiagThreads, smem, s>>>(
        Fd, W, d, rows_per_group, iters, C, Q, J, status);
    return cudaGetLastError();
}

cudaError_t lnq_diag_launch(const float *Fd, int groups, const float *W, int64_t d_out, int64_t d,
                            int m, int iters, float *C, uint8_t *Q, double *J, int32_t *status,
                            cudaStream_t s)
{
    const int64_t R = d_out / groups;
    switch (m) {
    case 2: return diag_m<2>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 4: return diag_m<4>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 8: return diag_m<8>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 16: return diag_m<16>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
