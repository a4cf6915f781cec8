// lnq_sweep.cu -- codebook solve, assignment sweep and objective of an LNQ iteration.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section: the codebook step
// c <- (P^T F P)^-1 P^T F w and the assignment step "for i = 1..d_in: give coordinate i the
// codeword minimising (w^ - w)^T F (w^ - w)".
//
// solve_kernel (one CTA per row). From V = F P and u = F r (lnq_vgemm.cu) it forms
// M = P^T V and t = P^T u in fp64. The coordinates are sorted by class first (a stable
// counting sort), and every sum runs in a fixed order, so results do not depend on scheduling.
// An fp64 Cholesky over the non-empty codewords then solves M dc = -t (the closed-form update in
// residual form), and the kernel writes c + dc in fp32 together with the exact fp32 change.
//
// sweep_kernel (one CTA per 32 rows of one group; lane = row). First u += V dc, so that u is
// F r for the new codebook. Then it walks blocks of 32 coordinates in order. One warp takes the
// block's decisions, coordinate after coordinate: candidate a changes the objective by
// Delta_a = delta_a (2 u_i + delta_a F_ii), the best strictly negative Delta moves the
// coordinate (lowest index on ties), and the block's later coordinates are corrected at once
// from the 32 x 32 diagonal tile of F. Then all warps apply the block's moves to every later
// coordinate, u[k] += sum_b delta_b F[k][b], skipping the update when no row moved.
//
// objective_kernel: J_j = r_j^T u_j with u = F r from the residual-only product, fp64 sums.
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kSolveThreads = 256;
constexpr int kSweepWarps = 8;
constexpr int kObjWarps = 8;
constexpr int kBlk = 32;

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
// assignment sweep
// ------------------------------------------------------------------------------------------
template <int M>
__global__ void __launch_bounds__(kSweepWarps * 32)
    sweep_kernel(const float *__restrict__ F, const float *__restrict__ V,
                 const float *__restrict__ dC, float *__restrict__ uT,
                 const float *__restrict__ C, uint8_t *__restrict__ Q, int64_t d, int64_t d_out,
                 int64_t rows_per_group, int blocks_per_group)
{
    __shared__ float c_s[kBlk][M + 1];
    __shared__ float fblk[kBlk][kBlk + 1];
    __shared__ __align__(16) float dl_s[kBlk][kBlk];
    __shared__ uint8_t qb_s[kBlk][kBlk + 4];
    __shared__ unsigned moved_s;  // bit ii: some row moved at coordinate b0 + ii

    const int g = blockIdx.x / blocks_per_group;
    const int rb = blockIdx.x - g * blocks_per_group;
    const int64_t gstart = static_cast<int64_t>(g) * rows_per_group;
    const int64_t row0 = gstart + static_cast<int64_t>(rb) * kBlk;
    const int64_t row_end = min(row0 + kBlk, gstart + rows_per_group);
    const float *Fg = F + static_cast<int64_t>(g) * d * d;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j = row0 + lane;
    const bool valid = j < row_end;

    for (int e = threadIdx.x; e < kBlk * M; e += blockDim.x) {
        const int r = e / M, b = e % M;
        c_s[r][b] = (row0 + r < row_end) ? C[(row0 + r) * M + b] : 0.f;
    }
    // 0. u <- u + V dc for every coordinate (u then equals F r for the new codebook)
    if (valid) {
        float dc[M];
#pragma unroll
        for (int b = 0; b < M; ++b)
            dc[b] = dC[j * M + b];
        const float *vj = V + j * d * M;
#pragma unroll 2
        for (int64_t k = warp; k < d; k += kSweepWarps) {
            const float *vk = vj + k * M;
            float acc = uT[k * d_out + j];
            if constexpr (M >= 4) {
#pragma unroll
                for (int b4 = 0; b4 < M / 4; ++b4) {
                    const float4 v4 = reinterpret_cast<const float4 *>(vk)[b4];
                    acc = fmaf(v4.x, dc[4 * b4], acc);
                    acc = fmaf(v4.y, dc[4 * b4 + 1], acc);
                    acc = fmaf(v4.z, dc[4 * b4 + 2], acc);
                    acc = fmaf(v4.w, dc[4 * b4 + 3], acc);
                }
            } else {
#pragma unroll
                for (int b = 0; b < M; ++b)
                    acc = fmaf(vk[b], dc[b], acc);
            }
            uT[k * d_out + j] = acc;
        }
    }
    __syncthreads();
    float c_reg[M];
#pragma unroll
    for (int b = 0; b < M; ++b)
        c_reg[b] = c_s[lane][b];

    for (int64_t b0 = 0; b0 < d; b0 += kBlk) {
        const int nb = (d - b0 < kBlk) ? static_cast<int>(d - b0) : kBlk;
        // stage the diagonal tile of F and the block's codeword indices
        for (int e = threadIdx.x; e < kBlk * kBlk; e += blockDim.x) {
            const int r = e / kBlk, c = e % kBlk;
            fblk[r][c] = (r < nb && c < nb) ? Fg[(b0 + r) * d + b0 + c] : 0.f;
            const int64_t jr = row0 + r;
            qb_s[r][c] = (jr < row_end && c < nb) ? (Q[jr * d + b0 + c] & (M - 1)) : 0;
        }
        __syncthreads();
        if (warp == 0) {
            float ub[kBlk];
#pragma unroll
            for (int ii = 0; ii < kBlk; ++ii)
                ub[ii] = (valid && ii < nb) ? uT[(b0 + ii) * d_out + j] : 0.f;
            unsigned colmask = 0u;
#pragma unroll
            for (int ii = 0; ii < kBlk; ++ii) {
                float dlt = 0.f;
                if (ii < nb && valid) {
                    const int qi = qb_s[lane][ii];
                    const float cur = c_s[lane][qi];
                    const float fii = fblk[ii][ii];
                    const float two_u = 2.f * ub[ii];
                    int best = qi;
                    float bestD = 0.f;
#pragma unroll
                    for (int a = 0; a < M; ++a) {
                        const float da = c_reg[a] - cur;
                        const float D = da * fmaf(da, fii, two_u);
                        if (D < bestD) {
                            bestD = D;
                            best = a;
                        }
                    }
                    if (best != qi) {  // a strictly negative Delta implies c[best] != cur
                        dlt = c_s[lane][best] - cur;
                        qb_s[lane][ii] = static_cast<uint8_t>(best);
                    }
                }
#pragma unroll
                for (int i2 = ii + 1; i2 < kBlk; ++i2)
                    ub[i2] = fmaf(dlt, fblk[ii][i2], ub[i2]);
                dl_s[ii][lane] = dlt;
                colmask |= (__ballot_sync(0xffffffffu, dlt != 0.f) != 0u ? 1u : 0u) << ii;
            }
            if (lane == 0)
                moved_s = colmask;
            if (valid && colmask != 0u) {
                for (int ii = 0; ii < nb; ++ii)
                    Q[j * d + b0 + ii] = qb_s[lane][ii];
            }
        }
        __syncthreads();
        const unsigned colmask = moved_s;
        if (colmask != 0u) {
            // Trailing update with one coordinate k per thread: the thread holds u[k] of the
            // block's 32 rows and F[k][b0..b0+31], and adds sum_ii delta[ii][row] F[k][b0+ii] over
            // the coordinates ii where some row moved (delta is read from shared memory as a
            // broadcast). Every thread has 64 independent loads in flight.
            const int nrows = static_cast<int>(row_end - row0);
            for (int64_t k = b0 + nb + threadIdx.x; k < d; k += blockDim.x) {
                float* urow = uT + k * d_out + row0;
                const float *frow = Fg + k * d + b0;
                float u[kBlk], f[kBlk];
                const bool vec_u = nrows == kBlk && (reinterpret_cast<uintptr_t>(urow) & 15u) == 0;
                const bool vec_f = nb == kBlk && (reinterpret_cast<uintptr_t>(frow) & 15u) == 0;
                if (vec_u) {
#pragma unroll
                    for (int v = 0; v < kBlk / 4; ++v) {
                        const float4 x = reinterpret_cast<const float4 *>(urow)[v];
                        u[4 * v] = x.x; u[4 * v + 1] = x.y; u[4 * v + 2] = x.z; u[4 * v + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < kBlk; ++r)
                        u[r] = r < nrows ? urow[r] : 0.f;
                }
                if (vec_f) {
#pragma unroll
                    for (int v = 0; v < kBlk / 4; ++v) {
                        const float4 x = reinterpret_cast<const float4 *>(frow)[v];
                        f[4 * v] = x.x; f[4 * v + 1] = x.y; f[4 * v + 2] = x.z; f[4 * v + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int ii = 0; ii < kBlk; ++ii)
                        f[ii] = ii < nb ? frow[ii] : 0.f;
                }
#pragma unroll
                for (int ii = 0; ii < kBlk; ++ii) {
                    if ((colmask >> ii) & 1u) {
                        const float fi = f[ii];
#pragma unroll
                        for (int v = 0; v < kBlk / 4; ++v) {
                            const float4 dd = *reinterpret_cast<const float4 *>(&dl_s[ii][4 * v]);
                            u[4 * v] = fmaf(dd.x, fi, u[4 * v]);
                            u[4 * v + 1] = fmaf(dd.y, fi, u[4 * v + 1]);
                            u[4 * v + 2] = fmaf(dd.z, fi, u[4 * v + 2]);
                            u[4 * v + 3] = fmaf(dd.w, fi, u[4 * v + 3]);
                        }
                    }
                }
                if (vec_u) {
#pragma unroll
                    for (int v = 0; v < kBlk / 4; ++v)
                        reinterpret_cast<float4 *>(urow)[v] =
                            make_float4(u[4 * v], u[4 * v + 1], u[4 * v + 2], u[4 * v + 3]);
                } else {
#pragma unroll
                    for (int r = 0; r < kBlk; ++r)
                        if (r < nrows)
                            urow[r] = u[r];
                }
            }
        }
        __syncthreads();
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

template <int M>
static cudaError_t sweep_m(const float *F, int groups, const float *V, const float *dC, float *uT,
                           const float *C, uint8_t *Q, int64_t d, int64_t d_out, cudaStream_t s)
{
    const int64_t R = d_out / groups;
    const int bpg = static_cast<int>((R + kBlk - 1) / kBlk);
    KernelTimer timer("lnq_sweep", s);
    sweep_kernel<M><<<static_cast<unsigned>(bpg * groups), kSweepWarps * 32, 0, s>>>(
        F, V, dC, uT, C, Q, d, d_out, R, bpg);
    return cudaGetLastError();
}

cudaError_t lnq_sweep(const float *F, int groups, const float *V, const float *dC, float *uT,
                      const float *C, uint8_t *Q, int64_t d, int64_t d_out, int m, cudaStream_t s)
{
    switch (m) {
    case 2: return sweep_m<2>(F, groups, V, dC, uT, C, Q, d, d_out, s);
    case 4: return sweep_m<4>(F, groups, V, dC, uT, C, Q, d, d_out, s);
    case 8: return sweep_m<8>(F, groups, V, dC, uT, C, Q, d, d_out, s);
    case 16: return sweep_m<16>(F, groups, V, dC, uT, C, Q, d, d_out, s);
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
