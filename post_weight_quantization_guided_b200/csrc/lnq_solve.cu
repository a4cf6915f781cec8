// lnq_solve.cu -- codebook solve and objective of an LNQ iteration.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section: the codebook step
// c <- (P^T F P)^-1 P^T F w, and the objective (w^ - w)^T F (w^ - w) of each row.
//
// solve_kernel (one CTA per row). From V = F P and U = -F w (lnq_vgemm.cu, the residual product
// with a zero codebook) it forms M = P^T V and t = P^T U = -P^T F w, streaming the row's V and U
// once with coalesced loads: fp32 partial sums over 32-coordinate chunks (a few terms each), fp64
// across chunks; every sum runs in a fixed order, so results do not depend on scheduling. An fp64
// Cholesky over the non-empty codewords (one warp, a lane per row) then solves M c = -t, the
// closed form c = (P^T F P)^-1 P^T F w, and the kernel writes the new codebook in fp32 to C and to
// dC (the sweep starts from u = U + V dC = F (c[q] - w)). Empty codewords keep their values; a
// singular M leaves the codebook unchanged.
//
// objective_u_kernel: J_j = r_j^T u_j with u = F r from the residual-only product, fp64 sums in a
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
    solve_kernel(const float *__restrict__ V, const float *__restrict__ U,
                 const uint8_t *__restrict__ Q, float *__restrict__ C, float *__restrict__ dC,
                 int32_t *__restrict__ status, int64_t d)
{
    constexpr int NW = kSolveThreads / 32;
    constexpr int PAIRS = M * M;
    constexpr int PPL = (PAIRS + 31) / 32;     // (class, column) pairs per lane, same class
    constexpr int LOGM = M == 2 ? 1 : (M == 4 ? 2 : (M == 8 ? 3 : 4));
    constexpr int SROW = M >= 4 ? M + 4 : 4;   // staged row: V[i][0..M-1], u[i]; 16-byte aligned
    __shared__ __align__(16) float stv[NW][32][SROW];  // staged V rows and u of 32 coordinates
    __shared__ uint8_t stq[NW][32];
    __shared__ double Mp[NW][PAIRS], tp[NW][M];
    __shared__ int cp[NW][M];
    __shared__ double Mm[PAIRS], tv[M], Ls[16][16];
    __shared__ int cnt[M];

    const int64_t j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *Vj = V + j * d * M;
    const float *Uj = U + j * d;
    const uint8_t *qj = Q + j * d;

    // 1. M[a][b] = sum over class-a coordinates of V[i][b], t[a] = sum of u[i], per warp in a
    //    fixed order: warp w takes 32-coordinate chunks w, w + NW, ...; a chunk is staged with
    //    coalesced loads, then lane (a, columns b0..b0+PPL) adds the staged rows of class a.
    const int p0 = lane * PPL;
    const bool owner = p0 < PAIRS;
    const int a = owner ? p0 / M : M;          // M: no class
    const int b0 = owner ? p0 % M : 0;
    double acc[PPL], tacc = 0.0;
    int n = 0;
#pragma unroll
    for (int q = 0; q < PPL; ++q)
        acc[q] = 0.0;
    const int64_t nch = (d + 31) / 32;
    for (int64_t ch = warp; ch < nch; ch += NW) {
        const int64_t i = ch * 32 + lane;
        if (i < d) {
            const float *vi = Vj + i * M;
            if constexpr (M >= 4) {
#pragma unroll
                for (int b4 = 0; b4 < M / 4; ++b4)
                    reinterpret_cast<float4 *>(&stv[warp][lane][0])[b4] =
                        reinterpret_cast<const float4 *>(vi)[b4];
            } else {
                const float2 x = *reinterpret_cast<const float2 *>(vi);
                stv[warp][lane][0] = x.x;
                stv[warp][lane][1] = x.y;
            }
            stv[warp][lane][M] = Uj[i];
            stq[warp][lane] = qj[i] & (M - 1);
        } else {
            stq[warp][lane] = 0xFF;
        }
        __syncwarp();
        // the chunk's coordinates of this lane's class (from one ballot per bit of the class),
        // visited in lane order: fp32 partials of the chunk, added to the fp64 sums once per chunk
        const int mq = stq[warp][lane];
        uint32_t mine = __ballot_sync(0xffffffffu, mq < M);
#pragma unroll
        for (int k = 0; k < LOGM; ++k) {
            const uint32_t bk = __ballot_sync(0xffffffffu, (mq >> k) & 1);
            mine &= ((a >> k) & 1) ? bk : ~bk;
        }
        if (!owner)
            mine = 0u;
        float pf[PPL], tf = 0.f;
#pragma unroll
        for (int q = 0; q < PPL; ++q)
            pf[q] = 0.f;
        n += __popc(mine);
        while (mine != 0u) {
            const int e = __ffs(mine) - 1;
            mine &= mine - 1u;
            if constexpr (PPL % 4 == 0) {
#pragma unroll
                for (int q4 = 0; q4 < PPL / 4; ++q4) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(&stv[warp][e][b0 + 4 * q4]);
                    pf[4 * q4] += v4.x;
                    pf[4 * q4 + 1] += v4.y;
                    pf[4 * q4 + 2] += v4.z;
                    pf[4 * q4 + 3] += v4.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < PPL; ++q)
                    pf[q] += stv[warp][e][b0 + q];
            }
            tf += stv[warp][e][M];
        }
#pragma unroll
        for (int q = 0; q < PPL; ++q)
            acc[q] += static_cast<double>(pf[q]);
        tacc += static_cast<double>(tf);
        __syncwarp();
    }
    if (owner) {
#pragma unroll
        for (int q = 0; q < PPL; ++q)
            Mp[warp][p0 + q] = acc[q];
        if (b0 == 0) {
            tp[warp][a] = tacc;
            cp[warp][a] = n;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < PAIRS; e += kSolveThreads) {
        double s = 0.0;
        for (int w = 0; w < NW; ++w)
            s += Mp[w][e];
        Mm[e] = s;
    }
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
        float *cn = dC + j * M;
        if (singular) {
            if (lane < M)
                cn[lane] = c[lane];
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
            if (lane < M)
                cn[lane] = c[lane];
            __syncwarp();
            if (lane < nn) {
                const float nw = static_cast<float>(x);
                c[myc] = nw;
                cn[myc] = nw;
            }
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
static cudaError_t solve_m(const float *V, const float *U, const uint8_t *Q, float *C, float *dC,
                           int32_t *status, int64_t d, int64_t d_out, cudaStream_t s)
{
    KernelTimer timer("lnq_solve", s);
    solve_kernel<M><<<static_cast<unsigned>(d_out), kSolveThreads, 0, s>>>(V, U, Q, C, dC, status, d);
    return cudaGetLastError();
}

cudaError_t lnq_solve(const float *V, const float *U, const uint8_t *Q, float *C, float *dC,
                      int32_t *status, int64_t d, int64_t d_out, int m, cudaStream_t s)
{
    switch (m) {
    case 2: return solve_m<2>(V, U, Q, C, dC, status, d, d_out, s);
    case 4: return solve_m<4>(V, U, Q, C, dC, status, d, d_out, s);
    case 8: return solve_m<8>(V, U, Q, C, dC, status, d, d_out, s);
    case 16: return solve_m<16>(V, U, Q, C, dC, status, d, d_out, s);
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
