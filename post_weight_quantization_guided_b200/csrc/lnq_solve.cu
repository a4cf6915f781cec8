// lnq_solve.cu -- codebook solve and objective of an LNQ iteration.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section: the codebook step
// c <- (P^T F P)^-1 P^T F w, and the objective (w^ - w)^T F (w^ - w) of each row.
//
// solve_kernel (one CTA per row). From V = F P and u = F r (lnq_vgemm.cu) it forms
// M = P^T V and t = P^T u in fp64. The coordinates are sorted by class first (a stable
// counting sort), and every sum runs in a fixed order, so results do not depend on scheduling.
// An fp64 Cholesky over the non-empty codewords then solves M dc = -t (the closed-form update in
// residual form), and the kernel writes c + dc in fp32 together with the exact fp32 change.
//
// objective_u_kernel: J_j = r_j^T u_j with u = F r from the residual-only product, fp64 sums.
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kSolveThreads = 256;
constexpr int kObjWarps = 8;

// ------------------------------------------------------------------------------------------
// codebook solve
// ------------------------------------------------------------------------------------------
template <int M>
__global__ void __launch_bounds__(kSolveThreads)
    solve_kernel(const float *__restrict__ V, const float *__restrict__ uT,
                 const uint8_t *__restrict__ Q, float *__restrict__ C, float *__restrict__ dC,
                 int32_t *__restrict__ status, int64_t d, int64_t d_out)
{
    constexpr int T = kSolveThreads;
    constexpr int PAIRS = M * M;
    constexpr int PPARTS = T / PAIRS;  // threads per (class, column) pair: 1, 4, 16, 64
    constexpr int TPARTS = T / M;      // threads per class for t
    extern __shared__ __align__(16) uint8_t sm[];
    int *cnt = reinterpret_cast<int *>(sm);               // [T][M] per-thread class counts
    int *list = cnt + T * M;                              // [d] class-sorted coordinates
    __shared__ int start[M + 1];
    __shared__ double Msum[PAIRS * PPARTS], tsum[M * TPARTS];
    __shared__ double Mm[M * M], tv[M], L[M * M], y[M];

    const int64_t j = blockIdx.x;
    const int tid = threadIdx.x;
    const uint8_t *q = Q + j * d;
    const int64_t chunk = (d + T - 1) / T;
    const int64_t lo = min(d, tid * chunk), hi = min(d, lo + chunk);

    // 1. stable counting sort of the coordinates by class
    for (int b = 0; b < M; ++b)
        cnt[tid * M + b] = 0;
    for (int64_t i = lo; i < hi; ++i)
        cnt[tid * M + (q[i] & (M - 1))] += 1;
    __syncthreads();
    if (tid < M) {  // exclusive scan over threads, per class
        int run = 0;
        for (int t = 0; t < T; ++t) {
            const int c = cnt[t * M + tid];
            cnt[t * M + tid] = run;
            run += c;
        }
        start[tid + 1] = run;  // class total, turned into starts below
    }
    __syncthreads();
    if (tid == 0) {
        start[0] = 0;
        for (int b = 0; b < M; ++b)
            start[b + 1] += start[b];
    }
    __syncthreads();
    {
        int off[M];
#pragma unroll
        for (int b = 0; b < M; ++b)
            off[b] = start[b] + cnt[tid * M + b];
        for (int64_t i = lo; i < hi; ++i) {
            const int b = q[i] & (M - 1);
#pragma unroll
            for (int bb = 0; bb < M; ++bb)
                if (bb == b)
                    list[off[bb]++] = static_cast<int>(i);
        }
    }
    __syncthreads();

    // 2. M[a][b] = sum_{i in class a} V[i][b], t[a] = sum_{i in class a} u[i]  (fp64, fixed order)
    {
        const int pair = tid / PPARTS, part = tid % PPARTS;
        const int a = pair / M, b = pair % M;
        double acc = 0.0;
        for (int e = start[a] + part; e < start[a + 1]; e += PPARTS)
            acc += static_cast<double>(V[(j * d + list[e]) * M + b]);
        Msum[pair * PPARTS + part] = acc;
        const int ta = tid / TPARTS, tpart = tid % TPARTS;
        double tacc = 0.0;
        for (int e = start[ta] + tpart; e < start[ta + 1]; e += TPARTS)
            tacc += static_cast<double>(uT[static_cast<int64_t>(list[e]) * d_out + j]);
        tsum[ta * TPARTS + tpart] = tacc;
    }
    __syncthreads();
    if (tid < PAIRS) {
        double s = 0.0;
        for (int part = 0; part < PPARTS; ++part)
            s += Msum[tid * PPARTS + part];
        Mm[tid] = s;
    }
    if (tid < M) {
        double s = 0.0;
        for (int part = 0; part < TPARTS; ++part)
            s += tsum[tid * TPARTS + part];
        tv[tid] = s;
    }
    __syncthreads();

    // 3. Cholesky over the non-empty codewords, dc = -M^-1 t
    if (tid == 0) {
        int idx[M];
        int nn = 0;
        for (int b = 0; b < M; ++b)
            if (start[b + 1] > start[b])
                idx[nn++] = b;
        bool singular = false;
        for (int r = 0; r < nn && !singular; ++r) {
            for (int c = 0; c <= r; ++c) {
                double s = Mm[idx[r] * M + idx[c]];
                for (int k = 0; k < c; ++k)
                    s -= L[r * M + k] * L[c * M + k];
                if (r == c) {
                    if (!(s > 0.0)) {
                        singular = true;
                        break;
                    }
                    L[r * M + r] = sqrt(s);
                } else {
                    L[r * M + c] = s / L[c * M + c];
                }
            }
        }
        float *c = C + j * M;
        float *dc = dC + j * M;
        for (int b = 0; b < M; ++b)
            dc[b] = 0.f;
        if (singular) {
            status[j] |= LNQ_ROW_SINGULAR;
        } else {
            for (int r = 0; r < nn; ++r) {
                double s = -tv[idx[r]];
                for (int k = 0; k < r; ++k)
                    s -= L[r * M + k] * y[k];
                y[r] = s / L[r * M + r];
            }
            for (int r = nn - 1; r >= 0; --r) {
                double s = y[r];
                for (int k = r + 1; k < nn; ++k)
                    s -= L[k * M + r] * y[k];
                y[r] = s / L[r * M + r];
            }
            for (int r = 0; r < nn; ++r) {
                const float old = c[idx[r]];
                const float nw = static_cast<float>(static_cast<double>(old) + y[r]);
                c[idx[r]] = nw;
                dc[idx[r]] = static_cast<float>(static_cast<double>(nw) - static_cast<double>(old));
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// objective J = r^T (F r)
// ------------------------------------------------------------------------------------------
template <int M>
__global__ void __launch_bounds__(kObjWarps * 32)
    objective_u_kernel(const float *__restrict__ uT, const float *__restrict__ W,
                       const float *__restrict__ C, const uint8_t *__restrict__ Q,
                       double *__restrict__ J, int64_t d, int64_t d_out)
{
    __shared__ double part[kObjWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + lane;
    double acc = 0.0;
    if (j < d_out) {
        for (int64_t i = warp; i < d; i += kObjWarps) {
            const float r = C[j * M + (Q[j * d + i] & (M - 1))] - W[j * d + i];
            acc += static_cast<double>(r) * static_cast<double>(uT[i * d_out + j]);
        }
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && j < d_out) {
        double s = 0.0;
        for (int w = 0; w < kObjWarps; ++w)
            s += part[w][lane];
        J[j] = s;
    }
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
template <int M>
static cudaError_t solve_m(const float *V, const float *uT, const uint8_t *Q, float *C, float *dC,
                           int32_t *status, int64_t d, int64_t d_out, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>(kSolveThreads) * M * 4 + static_cast<size_t>(d) * 4;
    cudaError_t e = cudaFuncSetAttribute(solve_kernel<M>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    KernelTimer timer("lnq_solve", s);
    solve_kernel<M><<<static_cast<unsigned>(d_out), kSolveThreads, smem, s>>>(V, uT, Q, C, dC,
                                                                              status, d, d_out);
    return cudaGetLastError();
}

cudaError_t lnq_solve(const float *V, const float *uT, const uint8_t *Q, float *C, float *dC,
                      int32_t *status, int64_t d, int64_t d_out, int m, cudaStream_t s)
{
    switch (m) {
    case 2: return solve_m<2>(V, uT, Q, C, dC, status, d, d_out, s);
    case 4: return solve_m<4>(V, uT, Q, C, dC, status, d, d_out, s);
    case 8: return solve_m<8>(V, uT, Q, C, dC, status, d, d_out, s);
    case 16: return solve_m<16>(V, uT, Q, C, dC, status, d, d_out, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t lnq_objective_from_u(const float *uT, const float *W, const float *C,
                                 const uint8_t *Q, double *J, int64_t d, int64_t d_out, int m,
                                 cudaStream_t s)
{
    const unsigned blocks = static_cast<unsigned>((d_out + 31) / 32);
    KernelTimer timer("lnq_objective", s);
    switch (m) {
    case 2: objective_u_kernel<2><<<blocks, kObjWarps * 32, 0, s>>>(uT, W, C, Q, J, d, d_out); break;
    case 4: objective_u_kernel<4><<<blocks, kObjWarps * 32, 0, s>>>(uT, W, C, Q, J, d, d_out); break;
    case 8: objective_u_kernel<8><<<blocks, kObjWarps * 32, 0, s>>>(uT, W, C, Q, J, d, d_out); break;
    case 16: objective_u_kernel<16><<<blocks, kObjWarps * 32, 0, s>>>(uT, W, C, Q, J, d, d_out); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace lnq
