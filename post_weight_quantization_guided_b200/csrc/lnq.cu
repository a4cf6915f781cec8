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
// The row's codebook from its sorted weights (the midpoint order statistics
// c_q = sorted[floor((2q+1) d / (2m))], read by `sorted_at`) and each weight's nearest codeword
// (fp64 distances, ties to the lower index).
template <typename SortedAt>
__device__ __forceinline__ void init_assign(const float *__restrict__ w, int64_t j, int64_t d, int m,
                                            float *__restrict__ C, uint8_t *__restrict__ Q,
                                            float *cb, SortedAt sorted_at)
{
    if (threadIdx.x < m) {
        const int64_t idx =
            (static_cast<int64_t>(2 * threadIdx.x + 1) * d) / (2 * static_cast<int64_t>(m));
        const float c = sorted_at(static_cast<int>(idx));
        cb[threadIdx.x] = c;
        C[j * m + threadIdx.x] = c;
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

// Rows shorter than 256 weights: bitonic sort of the padded row in shared memory.
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
    init_assign(w, j, d, m, C, Q, cb, [&](int idx) { return keys[idx]; });
}

// One in-thread stage of the register bitonic sort: compare-exchange positions k and k + S of the
// thread's K keys (S < K, a compile-time distance so the keys stay in registers).
template <int K, int S>
__device__ __forceinline__ void bitonic_in_thread(float (&v)[K], int base, int size)
{
    if constexpr (S < K) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if ((k & S) == 0) {
                const bool up = ((base + k) & size) == 0;
                const float a = v[k], b = v[k + S];
                const bool sw = (a > b) == up;
                v[k] = sw ? b : a;
                v[k + S] = sw ? a : b;
            }
        }
    }
}

// Rows of 256 weights or more: the same bitonic network over p2 = 256 K keys held in registers,
// thread t owning positions t K .. t K + K - 1. Compare-exchange partners at distance < K are in
// the thread, at distance < 32 K in the warp (shuffles); only the larger distances go through
// shared memory, stored transposed ([k][t], no bank conflicts). The sorted row is unique, so the
// result equals the shared-memory sort's.
template <int K>
__global__ void __launch_bounds__(kRowThreads) init_reg_kernel(const float *__restrict__ W,
                                                               int64_t d, int m,
                                                               float *__restrict__ C,
                                                               uint8_t *__restrict__ Q)
{
    constexpr int P2 = K * kRowThreads;
    extern __shared__ float xs[];  // [K][kRowThreads]
    __shared__ float cb[kMaxM];
    const int64_t j = blockIdx.x;
    const float *w = W + j * d;
    const int t = threadIdx.x;
    float v[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int64_t i = static_cast<int64_t>(t) * K + k;
        v[k] = (i < d) ? w[i] : __int_as_float(0x7f800000);  // +inf pads the tail
    }
    bool first_exchange = true;
    for (int size = 2; size <= P2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < K) {
                // partners in the thread
                switch (stride) {
                case 1: bitonic_in_thread<K, 1>(v, t * K, size); break;
                case 2: bitonic_in_thread<K, 2>(v, t * K, size); break;
                case 4: bitonic_in_thread<K, 4>(v, t * K, size); break;
                case 8: bitonic_in_thread<K, 8>(v, t * K, size); break;
                case 16: bitonic_in_thread<K, 16>(v, t * K, size); break;
                case 32: bitonic_in_thread<K, 32>(v, t * K, size); break;
                default: break;
                }
            } else {
                const int ts = stride / K;  // partner thread distance
                const bool lower = (t & ts) == 0;
                if (ts < 32) {
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const bool up = ((t * K + k) & size) == 0;
                        const float o = __shfl_xor_sync(0xffffffffu, v[k], ts);
                        v[k] = (lower == up) ? fminf(v[k], o) : fmaxf(v[k], o);
                    }
                } else {
                    if (!first_exchange)
                        __syncthreads();  // the previous exchange's reads are done
                    first_exchange = false;
#pragma unroll
                    for (int k = 0; k < K; ++k)
                        xs[k * kRowThreads + t] = v[k];
                    __syncthreads();
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const bool up = ((t * K + k) & size) == 0;
                        const float o = xs[k * kRowThreads + (t ^ ts)];
                        v[k] = (lower == up) ? fminf(v[k], o) : fmaxf(v[k], o);
                    }
                }
            }
        }
    }
    if (!first_exchange)
        __syncthreads();
#pragma unroll
    for (int k = 0; k < K; ++k)
        xs[k * kRowThreads + t] = v[k];
    __syncthreads();
    init_assign(w, j, d, m, C, Q, cb,
                [&](int idx) { return xs[(idx % K) * kRowThreads + idx / K]; });
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
    auto launch_reg = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        KernelTimer timer("lnq_init", s);
        kernel<<<static_cast<unsigned>(d_out), kRowThreads, smem, s>>>(W, d, m, C, Q);
        return cudaGetLastError();
    };
    switch (p2 / kRowThreads) {
    case 1: return launch_reg(init_reg_kernel<1>);
    case 2: return launch_reg(init_reg_kernel<2>);
    case 4: return launch_reg(init_reg_kernel<4>);
    case 8: return launch_reg(init_reg_kernel<8>);
    case 16: return launch_reg(init_reg_kernel<16>);
    case 32: return launch_reg(init_reg_kernel<32>);
    case 64: return launch_reg(init_reg_kernel<64>);
    default: break;
    }
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
    const int nhalves = static_cast<int>(2 * ((d + 255) / 256));
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
        // codebook step: M = P^T F P (binned over the upper block triangle), then the solve
        if ((e = lnq_vgemm(w.Fh, w.fexp, nullptr, groups, Q, W, C, w.Sb, nullptr, w.img, d, d_out,
                           m, false, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_solve(w.Sb, nhalves, w.U, Q, C, w.status, d, d_out, m, s)) != cudaSuccess)
            return e;
        // the sweep's starting u = F (c[q] - w) for the new codebook
        if ((e = lnq_residual_scale(Q, W, C, d, d_out, m, w.rexp, s)) != cudaSuccess)
            return e;
        if ((e = lnq_vgemm(w.Fh, w.fexp, w.rexp, groups, Q, W, C, nullptr, w.Ur, w.img, d, d_out,
                           m, true, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_sweep(F, w.Fh, w.fexp, groups, w.Ur, C, Q, w.hist, d, d_out, m, err, s)) !=
            cudaSuccess)
            return e;
    }
    if (J != nullptr) {
        if ((e = lnq_residual_scale(Q, W, C, d, d_out, m, w.rexp, s)) != cudaSuccess)
            return e;
        if ((e = lnq_vgemm(w.Fh, w.fexp, w.rexp, groups, Q, W, C, nullptr, w.Ur, w.img, d, d_out,
                           m, true, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_objective_from_u(w.Ur, W, C, Q, J, d, d_out, m, s)) != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

}  // namespace lnq
