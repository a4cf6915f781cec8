// ganq.cu -- a GANQ-style comparison solver for the same per-row problem, on sm_100a.
//
// Source: scime.ai summary of GANQ (GPU-adaptive non-uniform quantization), Approach paragraph:
// the per-row problem min (P c - w)^T F (P c - w) is solved by alternating a Cholesky /
// back-substitution assignment of the codebook indices with the closed-form least-squares
// codebook update, batched on the GPU. Here it is an A/B against LNQ's coordinate-descent sweep:
// the codebook step is LNQ's (lnq_vgemm + lnq_solve), only the assignment differs.
//
// Reading (the summary gives no more): the factor is lower, F = L L^T, so with r = c[q] - w the
// objective is ||L^T r||^2 = sum_i z_i^2, z_i = sum_{k >= i} L[k][i] r_k. Back-substitution
// visits i = d-1 down to 0 and gives coordinate i the codeword nearest to
// t_i = w_i - (sum_{k > i} L[k][i] r_k) / L[i][i] (the smallest |z_i| given the later
// coordinates); no damping or preconditioning. A group whose factorisation meets a non-positive
// pivot is not positive definite: its rows keep their codes (the codebook step still runs) and
// report LNQ_ROW_NOT_PD.
//
// Kernels:
//   chol_copy_kernel     F (fp32) -> A (fp64), every group.
//   chol_diag_kernel     right-looking blocked Cholesky in fp64, step k: the 32 x 32 diagonal
//                        block, one warp per group (lane = row of the block), in shared memory.
//   chol_panel_kernel    the panel below it: each thread one row, forward substitution with the
//                        block's factor.
//   chol_update_kernel   the trailing lower triangle minus the panel's outer product, in 64 x 64
//                        tiles (each thread 4 x 4 outputs, the two panel slices in shared memory).
//   chol_finish_kernel   L (fp32, zero above the diagonal) and 1 / L[i][i].
//   ganq_assign_kernel   16 rows of one group per CTA, coordinates in blocks of 32 from the last:
//                        (1) all 256 threads form s[row][i] = sum_{k past the block} L[k][i] r_k
//                        for the block's 32 coordinates (16 x 32 outputs, k in chunks of 128
//                        through a ring of three shared-memory stages filled by asynchronous
//                        copies, two chunks in flight while one is summed, fp32); (2) one warp (lane = row) decides the block from the
//                        last coordinate to the first, adding the block's own earlier decisions from
//                        its diagonal tile of L in registers, and finds the nearest codeword by a
//                        binary search of the sorted codebook's midpoints in registers; (3) the
//                        block's codes and residuals are written back (the residuals feed (1) of the
//                        blocks before it).
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kCholB = 32;       // panel width of the blocked factorisation
constexpr int kCholTile = 64;    // output tile of the trailing update
constexpr int kGanqRows = 16;    // rows per CTA of the assignment
constexpr int kGanqBlk = 32;     // coordinates per decision block
constexpr int kGanqThreads = 256;

__global__ void chol_copy_kernel(const float *__restrict__ F, int64_t total,
                                 double *__restrict__ A)
{
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x)
        A[e] = static_cast<double>(F[e]);
}

// Factor the nb x nb diagonal block at (k0, k0) of group blockIdx.x (nb <= 32). A non-positive
// pivot sets status[g] and leaves the rest of that group's factor undefined.
__global__ void __launch_bounds__(32) chol_diag_kernel(double *__restrict__ A, int64_t d,
                                                       int64_t k0, int32_t *__restrict__ status)
{
    __shared__ double a[kCholB][kCholB + 1];
    const int g = blockIdx.x, lane = threadIdx.x;
    double *Ag = A + static_cast<int64_t>(g) * d * d;
    const int nb = static_cast<int>(min(static_cast<int64_t>(kCholB), d - k0));
    for (int c = 0; c < nb; ++c)
        if (lane < nb)
            a[lane][c] = Ag[(k0 + lane) * d + k0 + c];
    __syncwarp();
    bool bad = false;
    for (int j = 0; j < nb; ++j) {
        if (lane == j) {
            const double piv = a[j][j];
            bad = !(piv > 0.0);
            a[j][j] = bad ? 1.0 : sqrt(piv);
        }
        bad = __any_sync(0xffffffffu, bad);
        __syncwarp();
        const double ljj = a[j][j];
        if (lane > j && lane < nb)
            a[lane][j] /= ljj;
        __syncwarp();
        if (lane > j && lane < nb) {
            const double lij = a[lane][j];
            for (int k = j + 1; k <= lane; ++k)
                a[lane][k] -= lij * a[k][j];
        }
        __syncwarp();
    }
    if (bad && lane == 0)
        status[g] = 1;
    for (int c = 0; c < nb; ++c)
        if (lane < nb && c <= lane)
            Ag[(k0 + lane) * d + k0 + c] = a[lane][c];
}

// Rows i >= k0 + nb of the panel: x = a_i L_kk^-T by forward substitution (one thread per row).
__global__ void __launch_bounds__(128) chol_panel_kernel(double *__restrict__ A, int64_t d,
                                                         int64_t k0)
{
    __shared__ double l[kCholB][kCholB + 1];
    const int g = blockIdx.y;
    double *Ag = A + static_cast<int64_t>(g) * d * d;
    const int nb = static_cast<int>(min(static_cast<int64_t>(kCholB), d - k0));
    for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) {
        const int r = e / nb, c = e % nb;
        l[r][c] = c <= r ? Ag[(k0 + r) * d + k0 + c] : 0.0;
    }
    __syncthreads();
    const int64_t i = k0 + nb + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= d)
        return;
    double x[kCholB];
#pragma unroll
    for (int c = 0; c < kCholB; ++c)
        x[c] = c < nb ? Ag[i * d + k0 + c] : 0.0;
#pragma unroll
    for (int c = 0; c < kCholB; ++c) {
        if (c < nb) {
            double v = x[c];
#pragma unroll
            for (int p = 0; p < c; ++p)
                v -= x[p] * l[c][p];
            x[c] = v / l[c][c];
        }
    }
#pragma unroll
    for (int c = 0; c < kCholB; ++c)
        if (c < nb)
            Ag[i * d + k0 + c] = x[c];
}

// Trailing update A[i][j] -= sum_p P[i][p] P[j][p] for k1 <= j <= i (tile pairs ti >= tj).
__global__ void __launch_bounds__(256) chol_update_kernel(double *__restrict__ A, int64_t d,
                                                          int64_t k0, int nb)
{
    __shared__ double pi[kCholTile][kCholB + 1];
    __shared__ double pj[kCholTile][kCholB + 1];
    const int g = blockIdx.y;
    double *Ag = A + static_cast<int64_t>(g) * d * d;
    const int64_t k1 = k0 + nb;
    // tile pair from the linear index: ti (ti + 1) / 2 + tj, tj <= ti
    const int64_t e = blockIdx.x;
    int64_t ti = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(e) + 1.0) - 1.0) / 2.0);
    while ((ti + 1) * (ti + 2) / 2 <= e)
        ++ti;
    while (ti * (ti + 1) / 2 > e)
        --ti;
    const int64_t tj = e - ti * (ti + 1) / 2;
    const int64_t i0 = k1 + ti * kCholTile, j0 = k1 + tj * kCholTile;
    for (int x = threadIdx.x; x < kCholTile * kCholB; x += blockDim.x) {
        const int r = x / kCholB, c = x % kCholB;
        pi[r][c] = (i0 + r < d && c < nb) ? Ag[(i0 + r) * d + k0 + c] : 0.0;
        pj[r][c] = (j0 + r < d && c < nb) ? Ag[(j0 + r) * d + k0 + c] : 0.0;
    }
    __syncthreads();
    const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            acc[a][b] = 0.0;
    for (int p = 0; p < nb; ++p) {
        double x[4], y[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            x[a] = pi[tr + a][p];
            y[a] = pj[tc + a][p];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
                acc[a][b] = fma(x[a], y[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t i = i0 + tr + a;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int64_t j = j0 + tc + b;
            if (i < d && j < d && j <= i)
                Ag[i * d + j] -= acc[a][b];
        }
    }
}

// L (fp32, zero above the diagonal) and 1 / L[i][i] from the fp64 factor.
__global__ void chol_finish_kernel(const double *__restrict__ A, int64_t d, int groups,
                                   float *__restrict__ L, float *__restrict__ invd)
{
    const int64_t total = static_cast<int64_t>(groups) * d * d;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t rc = e % (d * d), g = e / (d * d);
        const int64_t i = rc / d, j = rc % d;
        const double v = j <= i ? A[e] : 0.0;
        L[e] = static_cast<float>(v);
        if (i == j)
            invd[g * d + i] = static_cast<float>(1.0 / v);
    }
}

constexpr int kGanqKc = 128;     // k per chunk of step (1)
constexpr int kGanqLL = kGanqKc * kGanqBlk / 4 / kGanqThreads;     // float4 loads of L per thread
constexpr int kGanqRL = kGanqRows * kGanqKc / 4 / kGanqThreads;    // float4 loads of R per thread
constexpr int kGanqOut = kGanqRows * kGanqBlk / kGanqThreads;      // outputs of step (1) per thread
static_assert(kGanqLL * 4 * kGanqThreads == kGanqKc * kGanqBlk, "L chunk split");
static_assert(kGanqRL * 4 * kGanqThreads == kGanqRows * kGanqKc, "R chunk split");
static_assert(kGanqOut == 2, "two outputs per thread in step (1)");

constexpr int kGanqStages = 3;   // chunks in flight in step (1)
constexpr int kGanqRcLd = kGanqKc + 4;                               // row stride of a staged R chunk
constexpr int kGanqStage = kGanqKc * kGanqBlk + kGanqRows * kGanqRcLd;   // floats per stage
constexpr size_t kGanqSmem = static_cast<size_t>(kGanqStages) * kGanqStage * sizeof(float);

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One chunk of step (1) into a stage: L[kc + a][b0 .. b0 + 31] for a < kGanqKc (lc, [Kc][32])
// and R[j0 + row][kc .. kc + kGanqKc - 1] for the CTA's rows (rc, [rows][Kc + 4]); zeros past d
// and past the rows. kVec (d a multiple of 4): 16-byte asynchronous copies with zero fill;
// otherwise plain loads and stores.
template <bool kVec>
__device__ __forceinline__ void ganq_issue_chunk(float *stage, const float *__restrict__ Lg,
                                                 const float *__restrict__ R, int64_t d,
                                                 int64_t b0, int bw, int64_t j0, int nr,
                                                 int64_t kc)
{
    const int t = threadIdx.x;
    float *lc = stage;
    float *rc = stage + kGanqKc * kGanqBlk;
#pragma unroll
    for (int u = 0; u < kGanqLL; ++u) {
        const int e = t + kGanqThreads * u;
        const int a = e >> 3, c4 = (e & 7) * 4;   // L row a, columns c4 .. c4 + 3
        const int64_t k = kc + a;
        float *dst = lc + a * kGanqBlk + c4;
        const float *src = Lg + (k < d ? k : 0) * d + b0 + c4;
        if (kVec) {
            cp_async16_zfill(dst, k < d && c4 + 4 <= bw ? src : Lg, k < d && c4 + 4 <= bw);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                dst[c] = (k < d && c4 + c < bw) ? __ldg(src + c) : 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < kGanqRL; ++u) {
        const int e = t + kGanqThreads * u;
        const int row = e >> 5, k4 = (e & 31) * 4;   // R row, k offsets k4 .. k4 + 3
        const int64_t k = kc + k4;
        float *dst = rc + row * kGanqRcLd + k4;
        const float *src = R + (j0 + (row < nr ? row : 0)) * d + (k < d ? k : 0);
        if (kVec) {
            cp_async16_zfill(dst, row < nr && k + 4 <= d ? src : R, row < nr && k + 4 <= d);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                dst[c] = (row < nr && k + c < d) ? src[c] : 0.f;
        }
    }
}

template <int M, bool kVec>
__global__ void __launch_bounds__(kGanqThreads)
    ganq_assign_kernel(const float *__restrict__ L, const float *__restrict__ invd,
                       const int32_t *__restrict__ gstatus, const float *__restrict__ W,
                       const float *__restrict__ C, uint8_t *__restrict__ Q,
                       float *__restrict__ R, int32_t *__restrict__ status, int64_t d,
                       int64_t rows_per_group, int ctas_per_group)
{
    // step (1) uses the ring of chunk stages; steps (2) and (3) reuse the first stage's bytes for
    // ss, ws, rs and ld (barriers separate the steps)
    extern __shared__ __align__(16) float ganq_sm[];
    auto ss = reinterpret_cast<float(*)[kGanqBlk + 1]>(ganq_sm);           // s of the block
    auto ws = ss + kGanqRows;                                              // w of the block
    auto rs = ws + kGanqRows;                                              // r of the block
    auto ld = reinterpret_cast<float(*)[kGanqBlk]>(ganq_sm + 3 * kGanqRows * (kGanqBlk + 1));
    static_assert(3 * kGanqRows * (kGanqBlk + 1) + kGanqBlk * kGanqBlk <= kGanqStage,
                  "the decision tiles fit in one chunk stage");
    __shared__ float iv[kGanqBlk];                      // 1 / L[i][i] of the block
    __shared__ uint8_t qs[kGanqRows][kGanqBlk];
    const int g = blockIdx.x / ctas_per_group;
    const int64_t j0 = g * rows_per_group + static_cast<int64_t>(blockIdx.x % ctas_per_group) * kGanqRows;
    const int nr = static_cast<int>(min(static_cast<int64_t>(kGanqRows), (g + 1) * rows_per_group - j0));
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    if (gstatus[g] != 0) {          // not positive definite: codes kept
        if (t < nr)
            status[j0 + t] = LNQ_ROW_NOT_PD;
        return;
    }
    const float *Lg = L + static_cast<int64_t>(g) * d * d;
    // warp 0, lane = row: the sorted codebook, its codeword indices and midpoints in registers
    float sv[M], mid[M > 1 ? M - 1 : 1];
    uint32_t ordw[2] = {0u, 0u};     // sorted position -> codeword index, 4 bits each
    if (warp == 0) {
        const int r = lane < nr ? lane : 0;
        float cv[M];
#pragma unroll
        for (int a = 0; a < M; ++a)
            cv[a] = C[(j0 + r) * M + a];
#pragma unroll
        for (int a = 0; a < M; ++a) {
            int rank = 0;
#pragma unroll
            for (int b = 0; b < M; ++b)
                rank += (cv[b] < cv[a] || (cv[b] == cv[a] && b < a)) ? 1 : 0;
#pragma unroll
            for (int k = 0; k < M; ++k)
                if (k == rank)
                    sv[k] = cv[a];
            if (rank < 8)
                ordw[0] |= static_cast<uint32_t>(a) << (4 * rank);
            else
                ordw[1] |= static_cast<uint32_t>(a) << (4 * (rank - 8));
        }
#pragma unroll
        for (int k = 0; k + 1 < M; ++k)
            mid[k] = 0.5f * (sv[k] + sv[k + 1]);
    }
    const int64_t nblk = (d + kGanqBlk - 1) / kGanqBlk;
    for (int64_t blk = nblk - 1; blk >= 0; --blk) {
        const int64_t b0 = blk * kGanqBlk;
        const int bw = static_cast<int>(min(static_cast<int64_t>(kGanqBlk), d - b0));
        const int64_t kstart = b0 + bw;
        // (1) s[row][c] = sum_{k >= kstart} L[k][b0 + c] r[row][k]: chunks of kGanqKc through
        // shared memory, the next chunk's loads in flight while the current one is summed
        const int srow = t / (kGanqBlk / kGanqOut), scol = (t % (kGanqBlk / kGanqOut)) * kGanqOut;
        float acc[kGanqOut] = {0.f, 0.f};
        const int64_t nch = kstart < d ? (d - kstart + kGanqKc - 1) / kGanqKc : 0;
        // kGanqStages - 1 chunks in flight ahead of the one being summed; one commit group per
        // chunk slot (empty groups past the last chunk keep the count uniform)
#pragma unroll
        for (int c = 0; c < kGanqStages - 1; ++c) {
            if (c < nch)
                ganq_issue_chunk<kVec>(ganq_sm + c * kGanqStage, Lg, R, d, b0, bw, j0, nr,
                                       kstart + c * kGanqKc);
            cp_async_commit();
        }
        for (int64_t c = 0; c < nch; ++c) {
            cp_async_wait_group<kGanqStages - 2>();
            __syncthreads();    // chunk c visible; every thread is done with chunk c - 1
            const int64_t cn = c + kGanqStages - 1;
            if (cn < nch)
                ganq_issue_chunk<kVec>(ganq_sm + (cn % kGanqStages) * kGanqStage, Lg, R, d, b0, bw,
                                       j0, nr, kstart + cn * kGanqKc);
            cp_async_commit();
            const float *lc = ganq_sm + (c % kGanqStages) * kGanqStage;
            const float *rc = lc + kGanqKc * kGanqBlk;
#pragma unroll 4
            for (int k = 0; k < kGanqKc; k += 4) {
                const float4 r4 = *reinterpret_cast<const float4 *>(rc + srow * kGanqRcLd + k);
                const float rv[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float2 l2 =
                        *reinterpret_cast<const float2 *>(lc + (k + kk) * kGanqBlk + scol);
                    acc[0] = fmaf(rv[kk], l2.x, acc[0]);
                    acc[1] = fmaf(rv[kk], l2.y, acc[1]);
                }
            }
        }
        cp_async_wait_group<0>();
        __syncthreads();        // every thread is done with the stages before they are reused
#pragma unroll
        for (int c = 0; c < kGanqOut; ++c)
            ss[srow][scol + c] = acc[c];
        // the block's w, its diagonal tile of L and the reciprocal pivots
        for (int x = t; x < kGanqRows * kGanqBlk; x += kGanqThreads) {
            const int a = x / kGanqBlk, b = x % kGanqBlk;
            ws[a][b] = (a < nr && b < bw) ? W[(j0 + a) * d + b0 + b] : 0.f;
        }
        for (int x = t; x < kGanqBlk * kGanqBlk; x += kGanqThreads) {
            const int a = x / kGanqBlk, b = x % kGanqBlk;
            ld[a][b] = (a < bw && b < bw) ? Lg[(b0 + a) * d + b0 + b] : 0.f;
        }
        if (t < bw)
            iv[t] = invd[g * d + b0 + t];
        __syncthreads();
        // (2) decisions, last coordinate first
        if (warp == 0 && lane < kGanqRows) {
            float sacc[kGanqBlk];
#pragma unroll
            for (int c = 0; c < kGanqBlk; ++c)
                sacc[c] = 0.f;
#pragma unroll
            for (int c = kGanqBlk - 1; c >= 0; --c) {
                if (c < bw) {
                    const float s = ss[lane][c] + sacc[c];
                    const float w = ws[lane][c];
                    const float tt = w - s * iv[c];
                    float V[M], Mi[M];
                    uint32_t O[M];
#pragma unroll
                    for (int k = 0; k < M; ++k) {
                        V[k] = sv[k];
                        Mi[k] = k + 1 < M ? mid[k + 1 < M ? k : 0] : 0.f;
                        O[k] = (ordw[k >> 3] >> (4 * (k & 7))) & 0xFu;
                    }
#pragma unroll
                    for (int S = M; S > 1; S >>= 1) {
                        const int h = S / 2;
                        const bool up = tt > Mi[h - 1];
#pragma unroll
                        for (int k = 0; k < h; ++k) {
                            V[k] = up ? V[k + h] : V[k];
                            O[k] = up ? O[k + h] : O[k];
                        }
#pragma unroll
                        for (int k = 0; k + 1 < h; ++k)
                            Mi[k] = up ? Mi[k + h] : Mi[k];
                    }
                    const float r = V[0] - w;
                    rs[lane][c] = r;
                    qs[lane][c] = static_cast<uint8_t>(O[0]);
#pragma unroll
                    for (int e = 0; e < c; ++e)
                        sacc[e] = fmaf(ld[c][e], r, sacc[e]);
                }
            }
        }
        __syncthreads();
        // (3) codes and residuals of the block
        for (int x = t; x < kGanqRows * kGanqBlk; x += kGanqThreads) {
            const int a = x / kGanqBlk, b = x % kGanqBlk;
            if (a < nr && b < bw) {
                Q[(j0 + a) * d + b0 + b] = qs[a][b];
                R[(j0 + a) * d + b0 + b] = rs[a][b];
            }
        }
        __syncthreads();
    }
}

size_t lnq_ganq_extra_bytes(int64_t d, int64_t d_out, int groups)
{
    const size_t dd = static_cast<size_t>(d) * d * groups;
    return align_up(dd * 8, 256) + align_up(dd * 4, 256) +
           align_up(static_cast<size_t>(groups) * d * 4, 256) +
           align_up(static_cast<size_t>(d_out) * d * 4, 256) +
           align_up(static_cast<size_t>(groups) * 4, 256);
}

template <int M>
static cudaError_t ganq_assign_m(const float *L, const float *invd, const int32_t *gstatus,
                                 const float *W, const float *C, uint8_t *Q, float *R,
                                 int32_t *status, int64_t d, int64_t d_out, int groups,
                                 cudaStream_t s)
{
    const int64_t rpg = d_out / groups;
    const int cpg = static_cast<int>((rpg + kGanqRows - 1) / kGanqRows);
    KernelTimer timer("ganq_assign", s);
    auto launch = [&](auto kernel) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kGanqSmem));
        if (e != cudaSuccess)
            return e;
        kernel<<<static_cast<unsigned>(cpg) * groups, kGanqThreads, kGanqSmem, s>>>(
            L, invd, gstatus, W, C, Q, R, status, d, rpg, cpg);
        return cudaGetLastError();
    };
    return d % 4 == 0 ? launch(ganq_assign_kernel<M, true>) : launch(ganq_assign_kernel<M, false>);
}

cudaError_t lnq_ganq_launch(const float *F, int groups, const float *W, int64_t d_out, int64_t d,
                            int m, int iters, float *C, uint8_t *Q, double *J,
                            const LnqWorkspace &w, void *extra, DeviceErr err, int num_sms,
                            cudaStream_t s)
{
    cudaError_t e;
    const size_t dd = static_cast<size_t>(d) * d * groups;
    uint8_t *b = static_cast<uint8_t *>(extra);
    double *A = reinterpret_cast<double *>(b);
    b += align_up(dd * 8, 256);
    float *L = reinterpret_cast<float *>(b);
    b += align_up(dd * 4, 256);
    float *invd = reinterpret_cast<float *>(b);
    b += align_up(static_cast<size_t>(groups) * d * 4, 256);
    float *R = reinterpret_cast<float *>(b);
    b += align_up(static_cast<size_t>(d_out) * d * 4, 256);
    int32_t *gstatus = reinterpret_cast<int32_t *>(b);
    if (cudaMemsetAsync(gstatus, 0, static_cast<size_t>(groups) * 4, s) != cudaSuccess ||
        cudaMemsetAsync(R, 0, static_cast<size_t>(d_out) * d * 4, s) != cudaSuccess)
        return cudaErrorUnknown;
    if (iters > 0) {
        // the factors, once per call
        {
            KernelTimer timer("ganq_cholesky", s);
            chol_copy_kernel<<<num_sms * 8, 256, 0, s>>>(F, static_cast<int64_t>(dd), A);
            for (int64_t k0 = 0; k0 < d; k0 += kCholB) {
                const int nb = static_cast<int>(min(static_cast<int64_t>(kCholB), d - k0));
                chol_diag_kernel<<<groups, 32, 0, s>>>(A, d, k0, gstatus);
                const int64_t rest = d - k0 - nb;
                if (rest > 0) {
                    chol_panel_kernel<<<dim3(static_cast<unsigned>((rest + 127) / 128), groups), 128,
                                        0, s>>>(A, d, k0);
                    const int64_t T = (rest + kCholTile - 1) / kCholTile;
                    chol_update_kernel<<<dim3(static_cast<unsigned>(T * (T + 1) / 2), groups), 256,
                                         0, s>>>(A, d, k0, nb);
                }
            }
            chol_finish_kernel<<<num_sms * 8, 256, 0, s>>>(A, d, groups, L, invd);
        }
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        if ((e = lnq_split_f16(F, d, groups, w.Fh, w.fexp, s)) != cudaSuccess)
            return e;
        // U = -F w (the codebook step's right-hand side), shared by every iteration
        if ((e = lnq_residual_scale(Q, W, nullptr, d, d_out, m, w.rexp, s)) != cudaSuccess)
            return e;
        if ((e = lnq_vgemm(w.Fh, w.fexp, w.rexp, groups, Q, W, nullptr, nullptr, w.U, w.img, d,
                           d_out, m, true, err, num_sms, s)) != cudaSuccess)
            return e;
    } else if (J != nullptr) {
        if ((e = lnq_split_f16(F, d, groups, w.Fh, w.fexp, s)) != cudaSuccess)
            return e;
    }
    const int nhalves = static_cast<int>(2 * ((d + 255) / 256));
    for (int it = 0; it < iters; ++it) {
        if ((e = lnq_vgemm(w.Fh, w.fexp, nullptr, groups, Q, W, C, w.Sb, nullptr, w.img, d, d_out,
                           m, false, err, num_sms, s)) != cudaSuccess)
            return e;
        if ((e = lnq_solve(w.Sb, nhalves, w.U, Q, C, w.status, d, d_out, m, s)) != cudaSuccess)
            return e;
        switch (m) {
        case 2: e = ganq_assign_m<2>(L, invd, gstatus, W, C, Q, R, w.status, d, d_out, groups, s); break;
        case 4: e = ganq_assign_m<4>(L, invd, gstatus, W, C, Q, R, w.status, d, d_out, groups, s); break;
        case 8: e = ganq_assign_m<8>(L, invd, gstatus, W, C, Q, R, w.status, d, d_out, groups, s); break;
        case 16: e = ganq_assign_m<16>(L, invd, gstatus, W, C, Q, R, w.status, d, d_out, groups, s); break;
        default: e = cudaErrorInvalidValue;
        }
        if (e != cudaSuccess)
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
