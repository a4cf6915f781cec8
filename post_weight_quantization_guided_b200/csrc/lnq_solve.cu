// lnq_solve.cu -- codebook solve and objective of an LNQ iteration.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section: the codebook step
// c <- (P^T F P)^-1 P^T F w, and the objective (w^ - w)^T F (w^ - w) of each row.
//
// solve_kernel (one CTA per row). M = P^T F P is assembled from the class-binned partial sums of
// lnq_vgemm.cu (one m x m block S per 128 coordinates, over the upper block triangle of F):
// M = sum S + (sum S)^T, the sums in fp64 in a fixed order. t = P^T U = -P^T F w comes from
// U = -F w (the residual product with a zero codebook), streamed once with coalesced loads: fp32
// partial sums over 32-coordinate chunks, fp64 across chunks, in a fixed order. An fp64 Cholesky
// over the non-empty codewords (one warp, a lane per row) then solves M c = -t, the closed form
// c = (P^T F P)^-1 P^T F w, and the kernel writes the new codebook to C. Empty codewords keep
// their values; a singular M leaves the codebook unchanged.
//
// objective_u_kernel: J_j = r_j^T u_j with u = F r from the residual product, fp64 sums in a
// fixed order.
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kSolveThreads = 256;
constexpr int kObjThreads = 256;

// ------------------------------------------------------------------------------------------
// codebook solve
// ------------------------------------------------------------------------------------------
template <int M>
__global__ void __launch_bounds__(kSolveThreads)
    solve_kernel(const float *__restrict__ Sb, int nhalves, const float *__restrict__ U,
                 const uint8_t *__restrict__ Q, float *__restrict__ C,
                 int32_t *__restrict__ status, int64_t d, int64_t d_out)
{
    constexpr int NW = kSolveThreads / 32;
    constexpr int PAIRS = M * M;
    constexpr int LOGM = M == 2 ? 1 : (M == 4 ? 2 : (M == 8 ? 3 : 4));
    __shared__ float stu[NW][32];
    __shared__ uint8_t stq[NW][32];
    __shared__ double tp[NW][M];
    __shared__ int cp[NW][M];
    __shared__ double Ss[PAIRS], Mm[PAIRS], tv[M], Ls[16][16];
    __shared__ int cnt[M];

    const int64_t j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *Uj = U + j * d;
    const uint8_t *qj = Q + j * d;

    // 1a. S = sum over the coordinate halves of the binned blocks (fp64, halves in order)
    for (int e = threadIdx.x; e < PAIRS; e += kSolveThreads) {
        double acc = 0.0;
        for (int hh = 0; hh < nhalves; ++hh)
            acc += static_cast<double>(Sb[(static_cast<int64_t>(hh) * d_out + j) * PAIRS + e]);
        Ss[e] = acc;
    }
    // 1b. t[a] = sum over class-a coordinates of U, and the class counts, per warp in a fixed
    //     order: warp w takes 32-coordinate chunks w, w + NW, ...; lane a < M adds, in lane
    //     order, the staged u of the chunk's class-a coordinates.
    double tacc = 0.0;
    int n = 0;
    const int64_t nch = (d + 31) / 32;
    for (int64_t ch = warp; ch < nch; ch += NW) {
        const int64_t i = ch * 32 + lane;
        if (i < d) {
            stu[warp][lane] = Uj[i];
            stq[warp][lane] = qj[i] & (M - 1);
        } else {
            stq[warp][lane] = 0xFF;
        }
        __syncwarp();
        const int mq = stq[warp][lane];
        uint32_t mine = __ballot_sync(0xffffffffu, mq < M);
#pragma unroll
        for (int k = 0; k < LOGM; ++k) {
            const uint32_t bk = __ballot_sync(0xffffffffu, (mq >> k) & 1);
            mine &= ((lane >> k) & 1) ? bk : ~bk;
        }
        if (lane >= M)
            mine = 0u;
        float tf = 0.f;
        n += __popc(mine);
        while (mine != 0u) {
            const int e = __ffs(mine) - 1;
            mine &= mine - 1u;
            tf += stu[warp][e];
        }
        tacc += static_cast<double>(tf);
        __syncwarp();
    }
    if (lane < M) {
        tp[warp][lane] = tacc;
        cp[warp][lane] = n;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < PAIRS; e += kSolveThreads)
        Mm[e] = Ss[e] + Ss[(e % M) * M + e / M];   // M = S + S^T
    if (threadIdx.x < M) {
        double s = 0.0;
        int c = 0;
        for (int w = 0; w < NW; ++w) {
            s += tp[w][threadIdx.x];
            c += cp[w][threadIdx.x];
        }
        tv[threadIdx.x] = s;
        cnt[threadIdx.x] = c;
    }
    __syncthreads();

    // 2. Cholesky over the non-empty codewords (one warp, lane = row, right-looking), then
    //    c = -M^-1 t by forward and back substitution.
    if (warp == 0) {
        int idx[M];
        int nn = 0;
#pragma unroll
        for (int b = 0; b < M; ++b)
            if (cnt[b] > 0)
                idx[nn++] = b;
        const int myc = lane < nn ? idx[lane < M ? lane : 0] : 0;
        double arow[M];
#pragma unroll
        for (int c = 0; c < M; ++c)
            arow[c] = (lane < nn && c < nn) ? Mm[myc * M + idx[c]] : 0.0;
        bool singular = false;
#pragma unroll
        for (int k = 0; k < M; ++k) {
            if (k < nn && !singular) {
                const double piv = __shfl_sync(0xffffffffu, arow[k], k);
                if (!(piv > 0.0)) {
                    singular = true;
                } else {
                    const double lkk = sqrt(piv);
                    const double inv = 1.0 / lkk;
                    const double lik = lane > k ? arow[k] * inv : (lane == k ? lkk : 0.0);
                    arow[k] = lik;  // column k of the row now holds L[lane][k]
#pragma unroll
                    for (int jj = k + 1; jj < M; ++jj) {
                        if (jj < nn) {
                            const double ljk = __shfl_sync(0xffffffffu, lik, jj);
                            if (lane >= jj)
                                arow[jj] -= lik * ljk;
                        }
                    }
                }
            }
        }
        float *c = C + j * M;
        if (singular) {
            if (lane == 0)
                status[j] |= LNQ_ROW_SINGULAR;
        } else {
            if (lane < nn) {
#pragma unroll
                for (int k = 0; k < M; ++k)
                    Ls[lane][k] = (k <= lane) ? arow[k] : 0.0;
            }
            __syncwarp();
            // forward: L y = -t; lane r keeps its running sum
            double s = lane < nn ? -tv[myc] : 0.0;
            double y = 0.0;
            for (int k = 0; k < nn; ++k) {
                if (lane == k)
                    y = s / Ls[k][k];
                const double yk = __shfl_sync(0xffffffffu, y, k);
                if (lane > k && lane < nn)
                    s -= Ls[lane][k] * yk;
            }
            // back: L^T x = y
            s = y;
            double x = 0.0;
            for (int k = nn - 1; k >= 0; --k) {
                if (lane == k)
                    x = s / Ls[k][k];
                const double xk = __shfl_sync(0xffffffffu, x, k);
                if (lane < k)
                    s -= Ls[k][lane] * xk;
            }
            if (lane < nn)
                c[myc] = static_cast<float>(x);
        }
    }
}

// ------------------------------------------------------------------------------------------
// objective J = r^T (F r)
// ------------------------------------------------------------------------------------------
// One CTA per row: fp64 sum of r_i u_i over the row, each thread over a fixed stride of
// coordinates, then a fixed-order tree, so the result does not depend on scheduling.
template <int M>
__global__ void __launch_bounds__(kObjThreads)
    objective_u_kernel(const float *__restrict__ U, const float *__restrict__ W,
                       const float *__restrict__ C, const uint8_t *__restrict__ Q,
                       double *__restrict__ J, int64_t d)
{
    __shared__ double part[kObjThreads / 32];
    const int64_t j = blockIdx.x;
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < d; i += kObjThreads) {
        const float r = C[j * M + (Q[j * d + i] & (M - 1))] - W[j * d + i];
        acc += static_cast<double>(r) * static_cast<double>(U[j * d + i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        acc += __shfl_down_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0)
        part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < kObjThreads / 32; ++w)
            s += part[w];
        J[j] = s;
    }
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
template <int M>
static cudaError_t solve_m(const float *Sb, int nhalves, const float *U, const uint8_t *Q, float *C,
                           int32_t *status, int64_t d, int64_t d_out, cudaStream_t s)
{
    KernelTimer timer("lnq_solve", s);
    solve_kernel<M><<<static_cast<unsigned>(d_out), kSolveThreads, 0, s>>>(Sb, nhalves, U, Q, C,
                                                                          status, d, d_out);
    return cudaGetLastError();
}

cudaError_t lnq_solve(const float *Sb, int nhalves, const float *U, const uint8_t *Q, float *C,
                      int32_t *status, int64_t d, int64_t d_out, int m, cudaStream_t s)
{
    switch (m) {
    case 2: return solve_m<2>(Sb, nhalves, U, Q, C, status, d, d_out, s);
    case 4: return solve_m<4>(Sb, nhalves, U, Q, C, status, d, d_out, s);
    case 8: return solve_m<8>(Sb, nhalves, U, Q, C, status, d, d_out, s);
    case 16: return solve_m<16>(Sb, nhalves, U, Q, C, status, d, d_out, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t lnq_objective_from_u(const float *U, const float *W, const float *C,
                                 const uint8_t *Q, double *J, int64_t d, int64_t d_out, int m,
                                 cudaStream_t s)
{
    const unsigned blocks = static_cast<unsigned>(d_out);
    KernelTimer timer("lnq_objective", s);
    switch (m) {
    case 2: objective_u_kernel<2><<<blocks, kObjThreads, 0, s>>>(U, W, C, Q, J, d); break;
    case 4: objective_u_kernel<4><<<blocks, kObjThreads, 0, s>>>(U, W, C, Q, J, d); break;
    case 8: objective_u_kernel<8><<<blocks, kObjThreads, 0, s>>>(U, W, C, Q, J, d); break;
    case 16: objective_u_kernel<16><<<blocks, kObjThreads, 0, s>>>(U, W, C, Q, J, d); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace lnq
