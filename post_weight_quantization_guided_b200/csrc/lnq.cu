// lnq.cu -- LNQ (layer-wise non-uniform quantisation) per-row kernels on B200 (sm_100a).
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section. Row j has the problem
//   min_{P one-hot, c}  (P c - w_j)^T F_g (P c - w_j),
// and the iteration
//   repeat { codebook: c <- (P^T F P)^-1 P^T F w;
//            assignment: for i = 1..d_in, coordinate i takes the codeword minimising the objective }.
//
// The state between iterations is (C, Q): every iteration recomputes what it needs from
// (F, W, C, Q), and every reduction runs in a fixed order, so resuming from a saved (C, Q) is
// exact.
//
// This file holds the initialisation and the orchestration of an iteration:
//   init_kernel   sort w_j in shared memory (bitonic), pick the midpoint order statistics
//                 c_q = sorted[floor((2q+1) d / (2m))], assign each weight its nearest codeword
//                 (fp64 distances, ties to the lower index). One CTA per row.
//   once          residual lnq_vgemm with the zero codebook: U = -F w (P^T F w for every
//                 iteration's codebook, and u = F r = U + V c)
//   iteration     lnq_vgemm (V = F P on tensor cores) -> lnq_solve (codebook) -> lnq_sweep
//                 (assignment from u = U + V c); see lnq_vgemm.cu and lnq_sweep.cu.
//   objective     residual lnq_vgemm (u = F r) -> J = r^T u.
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kRowThreads = 256;
constexpr int kMaxM = 16;

// ------------------------------------------------------------------------------------------
// init
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kRowThreads) init_kernel(const float *__restrict__ W, int64_t d,
                                                           int m, float *__restrict__ C,
                                                           uint8_t *__restrict__ Q, int p2)
{
    extern __shared__ float keys[];  // [p2]
    __shared__ float cb[kMaxM];
    const int64_t j = blockIdx.x;
    const float *w = W + j * d;
    for (int i = threadIdx.x; i < p2; i += blockDim.x)
        keys[i] = (i < d) ? w[i] : __int_as_float(0x7f800000);  // +inf pads the tail
    __syncthreads();
    // Bitonic sort, ascending.
    for (int size = 2; size <= p2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < p2 / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = ((lo & size) == 0);
                const float a = keys[lo], b = keys[hi];
                if ((a > b) == up) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }
    if (threadIdx.x < m) {
        const int64_t idx = (static_cast<int64_t>(2 * threadIdx.x + 1) * d) / (2 * static_cast<int64_t>(m));
        cb[threadIdx.x] = keys[idx];
        C[j * m + threadIdx.x] = keys[idx];
    }
    __syncthreads();
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
        const double x = w[i];
        int best = 0;
        double bd = fabs(x - static_cast<double>(cb[0]));
        for (int a = 1; a < m; ++a) {
            const double dist = fabs(x - static_cast<double>(cb[a]));
            if (dist < bd) {
                bd = dist;
                best = a;
            }
        }
        Q[j * d + i] = static_cast<uint8_t>(best);
    }
}

}  // namespace lnq

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
namespace lnq {

cudaError_t lnq_init_launch(const float *W, int64_t d_out, int64_t d, int m, float *C,
                            uint8_t *Q, cudaStream_t s)
{
    int p2 = 1;
    while (p2 < d)
        p2 <<= 1;
    const size_t smem = static_cast<size_t>(p2) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(init_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    {
        KernelTimer timer("lnq_init", s);
        init_kernel<<<static_cast<unsigned>(d_out), kRowThreads, smem, s>>>(W, d, m, C, Q, p2);
    }
    return cudaGetLastError();
}

cudaError_t lnq_iterate_launch(const float *F, int groups, const float *W, int64_t d_out,
                               int64_t d, int m, int iters, float *C, uint8_t *Q, double *J,
                               const LnqWorkspace &w, DeviceErr err, int num_sms, cudaStream_t s)
{
    cudaError_t e;
    if (iters > 0 || J != nullptr)
        if ((e = lnq_split_f16(F, d, groups, w.Fh, w.fexp, s)) != cudaSuccess)
            return e;
    if (iters > 0) {
        // U = -F w (the residual of the zero codebook), shared by every iteration
        if ((e = lnq_residual_scale(Q, W, nullptr, d, d_out, m, w.rexp, s)) != cudaSuccess)
            return e;
        if ((e = lnq_vgemm(w.Fh, w.fexp, w.rexp, groups, Q, W, nullptr, nullptr, w.U, w.img, d,
                           d_out, m, true, err, num_sms, s)) != cudaSuccess)
            return e;
    }
    for (int it = 0; it < iters; ++it) {
        if ((e = lnq_vgemm(w.Fh, w.fexp, nullptr, groups, Q, W, C, w.V, nullptr, w.img, d, d_out,
                           m, false, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_solve(w.V, w.U, Q, C, w.dC, w.status, d, d_out, m, s)) != cudaSuccess)
            return e;
        if ((e = lnq_sweep(F, w.Fh, w.fexp, groups, w.V, w.dC, w.U, C, Q, w.hist, d, d_out, m,
                           err, s)) != cudaSuccess)
            return e;
    }
    if (J != nullptr) {
        if ((e = lnq_residual_scale(Q, W, C, d, d_out, m, w.rexp, s)) != cudaSuccess)
            return e;
        if ((e = lnq_vgemm(w.Fh, w.fexp, w.rexp, groups, Q, W, C, nullptr, w.U, w.img, d, d_out, m,
                           true, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_objective_from_u(w.U, W, C, Q, J, d, d_out, m, s)) != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

}  // namespace lnq
