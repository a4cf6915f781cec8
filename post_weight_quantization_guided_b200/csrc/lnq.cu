// lnq.cu -- LNQ (layer-wise non-uniform quantisation) per-row kernels on B200 (sm_100a).
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section. Row j has the problem
//   min_{P one-hot, c}  (P c - w_j)^T F_g (P c - w_j),
// and the iteration
//   repeat { codebook: c <- (P^T F P)^-1 P^T F w;
//            assignment: for i = 1..d_in, coordinate i takes the codeword minimising the objective }.
//
// The state between iterations is (C, Q); every kernel recomputes what it needs from
// (F, W, C, Q), so resuming from a saved (C, Q) is exact.
//
// Kernels (one CTA per row):
//   init_kernel      sort w_j in shared memory (bitonic), pick the midpoint order statistics
//                    c_q = sorted[floor((2q+1) d / (2m))], assign each weight its nearest codeword
//                    (fp64 distances, ties to the lower index).
//   codebook_kernel  one pass over F_g: warp per coordinate i, lanes over k (coalesced row of F).
//                    Per-lane class bins give V[i][b] = sum_{k: q_k = b} F[i][k]; with
//                    u_i = sum_k F[i][k] r_k they give M = P^T F P and t = P^T u in fp64. Then an
//                    fp64 Cholesky over the non-empty codewords solves M dc = -t (the closed-form
//                    update in residual form), and c <- c + dc.
//   sweep_kernel     u = F r (same pass shape), then coordinates i = 0..d-1 in order: candidate
//                    a changes the objective by Delta_a = delta_a (2 u_i + delta_a F_ii),
//                    delta_a = c_a - c_{q_i}; the best strictly negative Delta moves the coordinate
//                    (lowest index on ties) and u[k > i] += delta F[i][k].
//   objective_kernel J_j = r^T F r with fp32 products and fp64 sums.
#include "common.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kRowThreads = 256;
constexpr int kRowWarps = kRowThreads / 32;
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

// ------------------------------------------------------------------------------------------
// Shared pieces of the per-row kernels
// ------------------------------------------------------------------------------------------
struct RowArgs {
    const float *F;   // [groups][d][d]
    const float *W;   // [d_out][d]
    float *C;         // [d_out][m]
    uint8_t *Q;       // [d_out][d]
    int32_t *status;  // [d_out] sticky per-row status (workspace)
    double *J;        // [d_out] or nullptr
    int64_t d;
    int m;
    int64_t rows_per_group;
};

// Loads r = c[q] - w and q of row j into shared memory. Indices are read modulo m (m is a power
// of two), so a corrupt Q byte can never address outside the codebook.
__device__ __forceinline__ void load_residual(const RowArgs &a, int64_t j, const float *cb,
                                              float *rs, uint8_t *qs)
{
    const float *w = a.W + j * a.d;
    const uint8_t *q = a.Q + j * a.d;
    for (int64_t i = threadIdx.x; i < a.d; i += blockDim.x) {
        const uint8_t qi = static_cast<uint8_t>(q[i] & (a.m - 1));
        qs[i] = qi;
        rs[i] = cb[qi] - w[i];
    }
}

// Dot of row i of F with r: lanes stride over k, fp32 products and fp32 partial sums.
__device__ __forceinline__ float row_dot(const float *__restrict__ Fi, const float *rs, int64_t d,
                                         int lane)
{
    float acc = 0.f;
    for (int64_t k = lane; k < d; k += 32)
        acc = fmaf(Fi[k], rs[k], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// ------------------------------------------------------------------------------------------
// codebook step
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kRowThreads) codebook_kernel(RowArgs a)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int64_t d = a.d;
    const int m = a.m;
    const int64_t j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // layout: Mw [warps][m][m] f64 | tw [warps][m] f64 | bins [warps][m][32] f32 | rs [d] f32 | qs [d]
    double *Mw = reinterpret_cast<double *>(sm);
    double *tw = Mw + kRowWarps * m * m;
    float *bins = reinterpret_cast<float *>(tw + kRowWarps * m);
    float *rs = bins + kRowWarps * m * 32;
    uint8_t *qs = reinterpret_cast<uint8_t *>(rs + d);
    __shared__ float cb[kMaxM];
    __shared__ double M[kMaxM * kMaxM], t[kMaxM], L[kMaxM * kMaxM], y[kMaxM];
    __shared__ int cnt[kMaxM];

    const float *F = a.F + (j / a.rows_per_group) * d * d;
    if (threadIdx.x < m) {
        cb[threadIdx.x] = a.C[j * m + threadIdx.x];
        cnt[threadIdx.x] = 0;
    }
    for (int e = threadIdx.x; e < kRowWarps * m * m; e += blockDim.x)
        Mw[e] = 0.0;
    for (int e = threadIdx.x; e < kRowWarps * m; e += blockDim.x)
        tw[e] = 0.0;
    __syncthreads();
    load_residual(a, j, cb, rs, qs);
    __syncthreads();
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x)
        atomicAdd(&cnt[qs[i]], 1);

    float *mybins = bins + warp * m * 32;
    for (int64_t i = warp; i < d; i += kRowWarps) {
        for (int b = 0; b < m; ++b)
            mybins[b * 32 + lane] = 0.f;
        __syncwarp();
        const float *Fi = F + i * d;
        float uacc = 0.f;
        for (int64_t k = lane; k < d; k += 32) {
            const float f = Fi[k];
            mybins[qs[k] * 32 + lane] += f;
            uacc = fmaf(f, rs[k], uacc);
        }
        __syncwarp();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            uacc += __shfl_xor_sync(0xffffffffu, uacc, o);
        const int qi = qs[i];
        for (int b = 0; b < m; ++b) {
            float v = mybins[b * 32 + lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == b)
                Mw[(warp * m + qi) * m + b] += static_cast<double>(v);
        }
        if (lane == 0)
            tw[warp * m + qi] += static_cast<double>(uacc);
        __syncwarp();
    }
    __syncthreads();
    // Combine warps in a fixed order (deterministic).
    for (int e = threadIdx.x; e < m * m; e += blockDim.x) {
        double s = 0.0;
        for (int w = 0; w < kRowWarps; ++w)
            s += Mw[w * m * m + e];
        M[e] = s;
    }
    for (int e = threadIdx.x; e < m; e += blockDim.x) {
        double s = 0.0;
        for (int w = 0; w < kRowWarps; ++w)
            s += tw[w * m + e];
        t[e] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Cholesky of M restricted to the non-empty codewords; solve M dc = -t.
        int idx[kMaxM];
        int nn = 0;
        for (int b = 0; b < m; ++b)
            if (cnt[b] > 0)
                idx[nn++] = b;
        bool singular = false;
        for (int r = 0; r < nn && !singular; ++r) {
            for (int c = 0; c <= r; ++c) {
                double s = M[idx[r] * m + idx[c]];
                for (int k = 0; k < c; ++k)
                    s -= L[r * kMaxM + k] * L[c * kMaxM + k];
                if (r == c) {
                    if (!(s > 0.0)) {
                        singular = true;
                        break;
                    }
                    L[r * kMaxM + r] = sqrt(s);
                } else {
                    L[r * kMaxM + c] = s / L[c * kMaxM + c];
                }
            }
        }
        if (singular) {
            a.status[j] |= LNQ_ROW_SINGULAR;
        } else {
            for (int r = 0; r < nn; ++r) {
                double s = -t[idx[r]];
                for (int k = 0; k < r; ++k)
                    s -= L[r * kMaxM + k] * y[k];
                y[r] = s / L[r * kMaxM + r];
            }
            for (int r = nn - 1; r >= 0; --r) {
                double s = y[r];
                for (int k = r + 1; k < nn; ++k)
                    s -= L[k * kMaxM + r] * y[k];
                y[r] = s / L[r * kMaxM + r];
            }
            for (int r = 0; r < nn; ++r)
                a.C[j * m + idx[r]] = static_cast<float>(static_cast<double>(cb[idx[r]]) + y[r]);
        }
    }
}

// ------------------------------------------------------------------------------------------
// assignment sweep
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kRowThreads) sweep_kernel(RowArgs a)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int64_t d = a.d;
    const int m = a.m;
    const int64_t j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *us = reinterpret_cast<float *>(sm);     // [d]
    float *rs = us + d;                            // [d]
    uint8_t *qs = reinterpret_cast<uint8_t *>(rs + d);
    __shared__ float cb[kMaxM];
    __shared__ int s_move;
    __shared__ float s_delta;

    const float *F = a.F + (j / a.rows_per_group) * d * d;
    if (threadIdx.x < m)
        cb[threadIdx.x] = a.C[j * m + threadIdx.x];
    __syncthreads();
    load_residual(a, j, cb, rs, qs);
    __syncthreads();
    for (int64_t i = warp; i < d; i += kRowWarps) {
        const float u = row_dot(F + i * d, rs, d, lane);
        if (lane == 0)
            us[i] = u;
    }
    __syncthreads();

    for (int64_t i = 0; i < d; ++i) {
        const float *Fi = F + i * d;
        if (warp == 0) {
            const int qi = qs[i];
            const float ui = us[i];
            const float fii = Fi[i];
            float D = INFINITY;
            if (lane < m) {
                const float dl = cb[lane] - cb[qi];
                D = dl * fmaf(dl, fii, 2.f * ui);
            }
            // best = lowest lane with the minimum D
            float bD = D;
            int bl = lane;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float oD = __shfl_xor_sync(0xffffffffu, bD, o);
                const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
                if (oD < bD || (oD == bD && ol < bl)) {
                    bD = oD;
                    bl = ol;
                }
            }
            if (lane == 0) {
                const int mv = (bD < 0.f) ? bl : -1;
                s_move = mv;
                if (mv >= 0) {
                    s_delta = cb[mv] - cb[qi];
                    qs[i] = static_cast<uint8_t>(mv);
                }
            }
        }
        __syncthreads();
        if (s_move >= 0) {
            const float dl = s_delta;
            for (int64_t k = i + 1 + threadIdx.x; k < d; k += blockDim.x)
                us[k] = fmaf(dl, Fi[k], us[k]);
        }
        __syncthreads();
    }
    uint8_t *q = a.Q + j * d;
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x)
        q[i] = qs[i];
}

// ------------------------------------------------------------------------------------------
// objective
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kRowThreads) objective_kernel(RowArgs a)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int64_t d = a.d;
    const int m = a.m;
    const int64_t j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *rs = reinterpret_cast<float *>(sm);
    uint8_t *qs = reinterpret_cast<uint8_t *>(rs + d);
    __shared__ float cb[kMaxM];
    __shared__ double part[kRowWarps];
    const float *F = a.F + (j / a.rows_per_group) * d * d;
    if (threadIdx.x < m)
        cb[threadIdx.x] = a.C[j * m + threadIdx.x];
    __syncthreads();
    load_residual(a, j, cb, rs, qs);
    __syncthreads();
    double acc = 0.0;
    for (int64_t i = warp; i < d; i += kRowWarps) {
        const float *Fi = F + i * d;
        double s = 0.0;
        for (int64_t k = lane; k < d; k += 32)
            s += static_cast<double>(Fi[k] * rs[k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        acc += s * static_cast<double>(rs[i]);
    }
    if (lane == 0)
        part[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double J = 0.0;
        for (int w = 0; w < kRowWarps; ++w)
            J += part[w];
        a.J[j] = J;
    }
}

}  // namespace lnq

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
namespace lnq {

static size_t codebook_smem(int64_t d, int m)
{
    return static_cast<size_t>(kRowWarps) * m * m * 8 + static_cast<size_t>(kRowWarps) * m * 8 +
           static_cast<size_t>(kRowWarps) * m * 32 * 4 + static_cast<size_t>(d) * 5;
}
static size_t sweep_smem(int64_t d) { return static_cast<size_t>(d) * 9; }
static size_t objective_smem(int64_t d) { return static_cast<size_t>(d) * 5; }

static RowArgs row_args(const float *F, int groups, const float *W, int64_t d_out, int64_t d,
                        int m, float *C, uint8_t *Q, int32_t *status, double *J)
{
    RowArgs a;
    a.F = F;
    a.W = W;
    a.C = C;
    a.Q = Q;
    a.status = status;
    a.J = J;
    a.d = d;
    a.m = m;
    a.rows_per_group = d_out / groups;
    return a;
}

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
                               int32_t *status, cudaStream_t s)
{
    const RowArgs a = row_args(F, groups, W, d_out, d, m, C, Q, status, J);
    const size_t cb = codebook_smem(d, m), sw = sweep_smem(d), ob = objective_smem(d);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(codebook_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(cb))) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(sw))) != cudaSuccess)
        return e;
    for (int it = 0; it < iters; ++it) {
        {
            KernelTimer timer("lnq_codebook", s);
            codebook_kernel<<<static_cast<unsigned>(d_out), kRowThreads, cb, s>>>(a);
        }
        {
            KernelTimer timer("lnq_sweep", s);
            sweep_kernel<<<static_cast<unsigned>(d_out), kRowThreads, sw, s>>>(a);
        }
    }
    if (J != nullptr) {
        if ((e = cudaFuncSetAttribute(objective_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(ob))) != cudaSuccess)
            return e;
        KernelTimer timer("lnq_objective", s);
        objective_kernel<<<static_cast<unsigned>(d_out), kRowThreads, ob, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t lnq_objective_launch(const float *F, int groups, const float *W, const float *C,
                                 const uint8_t *Q, int64_t d_out, int64_t d, int m, double *J,
                                 cudaStream_t s)
{
    const RowArgs a = row_args(F, groups, W, d_out, d, m, const_cast<float *>(C),
                               const_cast<uint8_t *>(Q), nullptr, J);
    const size_t ob = objective_smem(d);
    cudaError_t e = cudaFuncSetAttribute(objective_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(ob));
    if (e != cudaSuccess)
        return e;
    {
        KernelTimer timer("lnq_objective", s);
        objective_kernel<<<static_cast<unsigned>(d_out), kRowThreads, ob, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace lnq
