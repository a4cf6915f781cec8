// lnq_vgemm.cu -- the dense contractions of an LNQ iteration on tcgen05 tensor cores.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section. The codebook update
// c <- (P^T F P)^-1 P^T F w needs, per output row j, the m x m matrix M_j = P_j^T F P_j (P_j the
// one-hot assignment, d x m), and the assignment sweep that follows starts from u_j = F r_j with
// r_j = c_j[q_j] - w_j. Both come from products of F with right operands that stack the rows of
// one Fisher group side by side, so that every row of the group shares the left operand F:
//
//   class-binned product (m > 0), over the upper block triangle only. With F = U + U^T, U the
//     blocks of 256 x 256 coordinates on and above the diagonal with the diagonal blocks halved,
//     M_j = P_j^T U P_j + (P_j^T U P_j)^T. For coordinate block I the product accumulates
//     V'_I = (1/2) F_II P_I + sum_{K > I} F_IK P_K (the diagonal block first; the first MMA of the
//     next block halves the accumulator exactly through its scale-input-d operand), and the
//     epilogue bins V'_I by class: S_I[q][.] = sum over coordinates i of I in class q of V'_I[i][.].
//     M_j is then the sum over I of S_I + S_I^T (lnq_solve.cu). Half of the dense product's work.
//   residual product (m == 0): u_j = F r_j for every row, r = c[q] - w (the zero codebook gives
//     -F w), used by the codebook's right-hand side, the sweep and the objective.
//
// Precision: each row i of F (fp32) is scaled by a power of two 2^fexp[i] that puts its largest
// entry in [2^14, 2^15) and split into two fp16 pieces H1 + H2 (22 significant bits of every
// entry). One-hot columns are exact in fp16 (two piece products). A residual row is scaled by
// 2^rexp[j] the same way and split into two fp16 pieces R1 + R2; three piece products
// H1 R1 + H1 R2 + H2 R1 (H2 R2 is below 2^-22 of each term, the size of the pieces' own rounding)
// accumulate in fp32 in TMEM, in segments of 8 K blocks whose sums the epilogue adds in fp32. The
// epilogues remove the power-of-two scales exactly.
//
// Two CTAs (a cluster pair on two SMs) share one MMA of 256 coordinates (i) x 256 columns: each CTA
// loads by TMA the F tiles of its own 128 coordinates and half (128 columns) of the right
// operand's tile (K-major, 128-byte swizzle, no multicast). The even CTA issues the MMAs; each
// CTA's TMEM holds its 128 coordinates x 256 columns, two accumulators alternating between tiles.
// The right operand of every (row tile, K block) is written once per product as an image in HBM:
//   one-hot: RT = 256 / m rows of m class columns;
//   residual: 128 rows; CTA h of the pair holds R1 of rows 64h .. 64h + 63, then their R2.
//   The H1 product takes all 256 columns; the H2 product takes only the R1 halves (N = 128) and
//   accumulates them 64 columns further on, into the R2 columns of the same rows.
#include <cuda_fp16.h>

#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

namespace vg {
constexpr int BM = 128;                          // coordinates per CTA; a pair covers 256
constexpr int PAIR_KB = 2 * BM / 64;             // K blocks per pair block of coordinates
constexpr int BK = 64;
constexpr int A_TILE = BM * BK * 2;              // one fp16 piece of a 128 x 64 F tile: 16 KB
constexpr int B_STAGES = 4;                      // right-operand half tiles in flight
constexpr int NUM_THREADS = 192;                 // w0 TMA, w1 MMA, w2-5 epilogue
constexpr int EPI_THREADS = 128;
constexpr int IP_BLOCK = 9;   // pair blocks per block of the tile order (see vg_tile_coords)
constexpr int EPI_BAR = 1;                       // named barrier of the epilogue warps
constexpr int TMEM_COLS = 512;
constexpr int NCOLS = 256;                       // MMA N: columns of the right operand per tile
constexpr int HALF = NCOLS / 2;                  // right-operand rows held by one CTA
constexpr int B_BYTES = HALF * 128;              // HALF rows x 64 k of 16-bit values: 16 KB
constexpr int VS_LD = 36;                        // floats per staged coordinate (32 + pad)
constexpr int VS_BYTES = BM * VS_LD * 4;         // one staged 32-column chunk: 18 KB
constexpr int MAX_DYN_SMEM = 232448;             // opt-in dynamic shared memory per block
constexpr int BAR_BYTES = 512;
constexpr uint16_t PAIR = 0x3;                   // both CTAs of the cluster
// After an error, how long a CTA lets its own copies land before the pair exits.
constexpr long long kPairDrainLimit = 1LL << 22;
}  // namespace vg

// Tile shapes. Both products take F as two fp16 pieces and the MMA is 256 columns wide, with two
// TMEM accumulators. The class-binned product (M > 0: RT = 256 / M rows of M one-hot columns per
// tile) accumulates a tile in one segment and its epilogue stages each 32-column chunk in shared
// memory (two buffers) next to the tile's codes; the residual product (M == 0: 128 rows per tile)
// accumulates segments of SEGK K blocks, which its epilogue adds into fp32 sums per row held in
// registers.
template <int M>
struct VgShape {
    static constexpr int PIECES = 2;                    // fp16 pieces of F in the left operand
    static constexpr int SEGK = M > 0 ? 0 : 8;          // K blocks per segment (0: whole tile)
    static constexpr int SETS = 2;                      // accumulators
    static constexpr int RT = M > 0 ? vg::NCOLS / M : 128;  // rows per tile
    static constexpr int EPI_BYTES = M > 0 ? 2 * vg::VS_BYTES + RT * vg::BM : 0;
    static constexpr int A_FIT = (vg::MAX_DYN_SMEM - 1024 - vg::BAR_BYTES -
                                  vg::B_STAGES * vg::B_BYTES - EPI_BYTES) / vg::A_TILE;
    static constexpr int A_SLOTS = A_FIT < 12 ? A_FIT : 12;
    static constexpr size_t SMEM = 1024 + static_cast<size_t>(A_SLOTS) * vg::A_TILE +
                                   vg::B_STAGES * vg::B_BYTES + EPI_BYTES + vg::BAR_BYTES;
    static_assert(SETS * vg::NCOLS <= vg::TMEM_COLS, "TMEM holds 512 fp32 columns");
    static_assert(A_SLOTS >= 2 * PIECES, "at least two K blocks of F in flight");
    static_assert(A_SLOTS <= 32, "slot phases are kept in 32-bit masks");
    static_assert(SMEM <= vg::MAX_DYN_SMEM, "shared memory");
    static_assert(M == 0 || (M <= 32 && (32 / (M > 0 ? M : 1)) * M == 32), "a 32-column chunk holds whole rows");
};

// Row stride (elements) of the fp16 pieces of F: TMA needs row strides that are multiples of 16 B.
__host__ __device__ inline int64_t pieces_stride(int64_t d) { return (d + 7) / 8 * 8; }

// F (fp32 [groups][d][d]) -> Fh (fp16 [groups][2][d][ld]) with a power-of-two scale per row:
// F[i][k] 2^fexp[i] = H1 + H2 up to 2^-22 relative (2^-39 of the row's largest entry for entries
// near the fp16 subnormal range), the row's largest entry scaled into [2^14, 2^15). One CTA per
// row. The epilogue of the product multiplies by 2^-fexp[i], exactly.
__global__ void __launch_bounds__(256)
    split_f16_kernel(const float *__restrict__ F, int64_t d, __half *__restrict__ Fh,
                     int32_t *__restrict__ fexp)
{
    __shared__ float red[8];
    const int64_t row = blockIdx.x;            // g * d + i
    const int64_t g = row / d, i = row - g * d;
    const float *src = F + row * d;
    float mx = 0.f;
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x)
        mx = fmaxf(mx, fabsf(src[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w)
        mx = fmaxf(mx, red[w]);
    const int s = mx > 0.f ? clamp_scale(14 - ilogbf(mx)) : 0;
    if (threadIdx.x == 0)
        fexp[row] = s;
    const float sc = pow2f(s);
    const int64_t ld = pieces_stride(d);
    __half *h1 = Fh + (g * 2 * d + i) * ld;
    __half *h2 = h1 + d * ld;
    for (int64_t k = threadIdx.x; k < ld; k += blockDim.x) {
        float x = 0.f;
        if (k < d)
            x = src[k] * sc;
        const __half a = __float2half_rn(x);
        h1[k] = a;
        h2[k] = __float2half_rn(x - __half2float(a));
    }
}

// Per-row power-of-two scale of the residual r_j = c_j[q_j] - w_j for the fp16 right operand:
// max_k |r_jk| 2^rexp[j] in [2^14, 2^15); C == nullptr stands for the zero codebook (r_j = -w_j).
// One warp per row.
__global__ void __launch_bounds__(256)
    residual_scale_kernel(const uint8_t *__restrict__ Q, const float *__restrict__ W,
                          const float *__restrict__ C, int64_t d, int64_t d_out, int m,
                          int32_t *__restrict__ rexp)
{
    const int64_t j = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= d_out)
        return;
    float mx = 0.f;
    for (int64_t k = lane; k < d; k += 32)
        mx = fmaxf(mx, fabsf((C != nullptr ? C[j * m + (Q[j * d + k] & (m - 1))] : 0.f) - W[j * d + k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0)
        rexp[j] = mx > 0.f ? clamp_scale(14 - ilogbf(mx)) : 0;
}


// The right operand of every (row tile, K block), written once per product and then loaded by TMA
// like F: NCOLS rows (the product's columns) x 64 coordinates, row-major
// [row tiles][K blocks][NCOLS][64], fp16. One-hot image (M > 0): row n of a row tile is the
// indicator of class n % M for the tile's row n / M. Residual image (M == 0): rows 128 h .. 128 h +
// 63 hold piece R1 of the tile's rows 64 h .. 64 h + 63 and rows 128 h + 64 .. 128 h + 127 their R2
// (h = 0, 1: the half each CTA of the pair loads). Everything outside the problem is zero.

// The one-hot image with one task per (row tile, row, 8 coordinates): the task reads its 8 codes
// once and writes its row's M class columns (16 bytes each; a warp's 32 tasks cover 4 rows x 64
// coordinates, so each class store fills 4 whole 128-byte rows of the image).
template <int M>
__global__ void __launch_bounds__(256)
    onehot_image_kernel(const uint8_t *__restrict__ Q, int64_t d, int64_t rows_per_group,
                        int row_tiles_per_group, int64_t ntasks, int nk, uint16_t *__restrict__ img)
{
    using S = VgShape<M>;
    static_assert(M > 0 && S::RT * M == vg::NCOLS, "one-hot columns fill the tile");
    const bool vec = (d & 7) == 0 && (reinterpret_cast<uintptr_t>(Q) & 7u) == 0;
    for (int64_t task = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; task < ntasks;
         task += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(task & 7);
        const int r = static_cast<int>((task >> 3) % S::RT);
        const int64_t tb = (task >> 3) / S::RT;
        const int kb = static_cast<int>(tb % nk);
        const int rt_all = static_cast<int>(tb / nk);
        const int g = rt_all / row_tiles_per_group;
        const int rt = rt_all - g * row_tiles_per_group;
        const int64_t gstart = static_cast<int64_t>(g) * rows_per_group;
        const int64_t j = gstart + static_cast<int64_t>(rt) * S::RT + r;
        const int64_t k0 = static_cast<int64_t>(kb) * 64 + 8 * c;
        uint8_t qv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            qv[e] = 0xFFu;  // no class: outside the problem
        if (j < gstart + rows_per_group && k0 < d) {
            if (vec && k0 + 8 <= d) {
                const uint2 q2 = *reinterpret_cast<const uint2 *>(Q + j * d + k0);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    qv[e] = static_cast<uint8_t>(q2.x >> (8 * e));
                    qv[4 + e] = static_cast<uint8_t>(q2.y >> (8 * e));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (k0 + e < d)
                        qv[e] = Q[j * d + k0 + e];
            }
        }
        uint16_t *dst = img + (tb * vg::NCOLS + static_cast<int64_t>(r) * M) * 64 + 8 * c;
#pragma unroll
        for (int b = 0; b < M; ++b) {
            uint32_t out[4];
#pragma unroll
            for (int h = 0; h < 4; ++h)
                out[h] = (qv[2 * h] == b ? 0x3C00u : 0u) | ((qv[2 * h + 1] == b ? 0x3C00u : 0u) << 16);
            *reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(b) * 64) =
                make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

// The residual image with one task per (row tile, row, 8 coordinates): the task forms its 8
// residuals r = c[q] - w (C == nullptr: r = -w) once, scales them by 2^rexp of the row and writes
// the two fp16 pieces R1 = fp16(r), R2 = fp16(r - R1) (16 bytes each).
__global__ void __launch_bounds__(256)
    residual_image_kernel(const uint8_t *__restrict__ Q, const float *__restrict__ W,
                          const float *__restrict__ C, const int32_t *__restrict__ rexp, int64_t d,
                          int64_t rows_per_group, int row_tiles_per_group, int64_t ntasks, int nk,
                          int m, uint16_t *__restrict__ img)
{
    constexpr int RT = VgShape<0>::RT;
    const bool vec = (d & 7) == 0 && (reinterpret_cast<uintptr_t>(Q) & 7u) == 0 &&
                     (reinterpret_cast<uintptr_t>(W) & 15u) == 0;
    for (int64_t task = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; task < ntasks;
         task += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(task & 7);
        const int r = static_cast<int>((task >> 3) % RT);
        const int64_t tb = (task >> 3) / RT;
        const int kb = static_cast<int>(tb % nk);
        const int rt_all = static_cast<int>(tb / nk);
        const int g = rt_all / row_tiles_per_group;
        const int rt = rt_all - g * row_tiles_per_group;
        const int64_t gstart = static_cast<int64_t>(g) * rows_per_group;
        const int64_t j = gstart + static_cast<int64_t>(rt) * RT + r;
        const int64_t k0 = static_cast<int64_t>(kb) * 64 + 8 * c;
        uint32_t out[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
        if (j < gstart + rows_per_group && k0 < d) {
            uint8_t qv[8];
            float wv[8];
            if (vec && k0 + 8 <= d) {
                const uint2 q2 = *reinterpret_cast<const uint2 *>(Q + j * d + k0);
                const float4 w0 = *reinterpret_cast<const float4 *>(W + j * d + k0);
                const float4 w1 = *reinterpret_cast<const float4 *>(W + j * d + k0 + 4);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    qv[e] = static_cast<uint8_t>(q2.x >> (8 * e));
                    qv[4 + e] = static_cast<uint8_t>(q2.y >> (8 * e));
                }
                wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
                wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const bool in = k0 + e < d;
                    qv[e] = in ? Q[j * d + k0 + e] : 0xFFu;
                    wv[e] = in ? W[j * d + k0 + e] : 0.f;
                }
            }
            const float sc = pow2f(rexp[j]);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (qv[e] == 0xFFu)
                    continue;
                const float rv = ((C != nullptr ? C[j * m + (qv[e] & (m - 1))] : 0.f) - wv[e]) * sc;
                const __half p1 = __float2half_rn(rv);
                const __half p2 = __float2half_rn(rv - __half2float(p1));
                const int sh = 16 * (e & 1);
                out[0][e >> 1] |= static_cast<uint32_t>(__half_as_ushort(p1)) << sh;
                out[1][e >> 1] |= static_cast<uint32_t>(__half_as_ushort(p2)) << sh;
            }
        }
        const int base_row = (r >> 6) * vg::HALF + (r & 63);
        uint16_t *dst = img + (tb * vg::NCOLS + base_row) * 64 + 8 * c;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc)
            *reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(pc) * 64 * 64) =
                make_uint4(out[pc][0], out[pc][1], out[pc][2], out[pc][3]);
    }
}

struct VgParams {
    const uint8_t *Q;   // [d_out][d]
    float *S;           // [2 i_pairs][d_out][m][m] class-binned partial sums (m > 0)
    float *U;           // [d_out][d] u = F r per row (m == 0)
    const int32_t *fexp;  // [groups][d] row scales of the fp16 pieces of F
    const int32_t *rexp;  // [d_out] residual scales
    int64_t d, d_out, rows_per_group;
    int row_tiles_per_group, i_pairs, num_tiles;
    DeviceErr err;
};

// Tile -> (group, rows [row0, row_end), coordinate pair block ip, row tile rt_all over all
// groups). Within a group the tiles run in blocks of IP_BLOCK pair blocks: row tile by row tile,
// and within a row tile the block's pair blocks. The pairs running at the same time then cover
// about 8 row tiles x IP_BLOCK pair blocks of one group: each F piece tile is read by the 8 row
// tiles at once and each right-operand tile by the IP_BLOCK pair blocks, so both come from L2
// after their first read even when a group's F pieces (2 d^2 x 2 bytes) are far larger than L2.
template <int M>
__device__ __forceinline__ void vg_tile_coords(const VgParams &p, int tile, int &g, int64_t &row0,
                                               int64_t &row_end, int &ip, int &rt_all)
{
    constexpr int RT = VgShape<M>::RT;
    const int per_group = p.row_tiles_per_group * p.i_pairs;
    g = tile / per_group;
    int o = tile - g * per_group;
    const int full = p.i_pairs / vg::IP_BLOCK;               // whole blocks of pair blocks
    const int per_full = p.row_tiles_per_group * vg::IP_BLOCK;
    int ipb, width;
    if (o < full * per_full) {
        ipb = o / per_full;
        o -= ipb * per_full;
        width = vg::IP_BLOCK;
    } else {
        ipb = full;
        o -= full * per_full;
        width = p.i_pairs - full * vg::IP_BLOCK;
    }
    const int rt = o / width;
    ip = ipb * vg::IP_BLOCK + (o - rt * width);
    rt_all = g * p.row_tiles_per_group + rt;
    const int64_t gstart = static_cast<int64_t>(g) * p.rows_per_group;
    row0 = gstart + static_cast<int64_t>(rt) * RT;
    row_end = min(row0 + RT, gstart + p.rows_per_group);
}

// First K block of a tile: the class-binned product covers the upper block triangle (K blocks of
// the diagonal pair block and beyond), the residual product all of K.
template <int M>
__device__ __forceinline__ int vg_first_kb(int ip) { return M > 0 ? ip * vg::PAIR_KB : 0; }

template <int M>
__global__ void __launch_bounds__(vg::NUM_THREADS, 1)
    lnq_vgemm_kernel(const __grid_constant__ CUtensorMap fmap, const __grid_constant__ CUtensorMap bmap,
                     VgParams p)
{
    using namespace vg;
    using S = VgShape<M>;
    constexpr int NSLOT = S::A_SLOTS;
    constexpr uint32_t IDESC = umma_idesc_f16kind(2 * BM, NCOLS, false, false, true);
    constexpr uint32_t IDESC_R1 = umma_idesc_f16kind(2 * BM, NCOLS / 2, false, false, true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t *a_base = smem;                                       // [NSLOT][16 KB]
    uint8_t *b_base = smem + NSLOT * A_TILE;                      // [B_STAGES][B_BYTES]
    uint8_t *e_base = b_base + B_STAGES * B_BYTES;                // epilogue staging (M > 0)
    uint64_t *bars = reinterpret_cast<uint64_t *>(e_base + S::EPI_BYTES);
    uint64_t *a_full = bars;                                      // [NSLOT] (the even CTA's count)
    uint64_t *a_empty = a_full + NSLOT;                           // [NSLOT]
    uint64_t *b_full = a_empty + NSLOT;                           // [B_STAGES] (the even CTA's count)
    uint64_t *b_empty = b_full + B_STAGES;                        // [B_STAGES]
    uint64_t *tfull = b_empty + B_STAGES;                         // [SETS]
    uint64_t *tempty = tfull + S::SETS;                           // [SETS] (even CTA's count)
    uint64_t *drain = tempty + S::SETS;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cr = cluster_ctarank();  // 0: issues the pair's MMAs; 1: its peer
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int a = 0; a < S::SETS; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * EPI_THREADS);     // the epilogues of both CTAs
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&fmap);
        tma_prefetch_desc(&bmap);
    }
    if (warp == 1)
        tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int nk = static_cast<int>((p.d + BK - 1) / BK);
    const long long limit = p.err.limit;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA: operands
        // Per K block: this CTA's half of the right-operand tile (HALF rows of the operand image),
        // then one 16 KB piece tile of F for this CTA's 128 coordinates per slot. The bytes of both
        // CTAs are counted on the even CTA's barriers (armed by its thread for both), and the even
        // CTA's MMA commits release stages and slots in both CTAs.
        if (lane == 0) {
            int slot = 0, bs = 0;
            uint32_t apar = 0u, aused = 0u, bpar = 0u, bused = 0u;  // parity of fills, ever filled
            bool ok = true;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, ip, rt_all;
                int64_t row0, row_end;
                vg_tile_coords<M>(p, tile, g, row0, row_end, ip, rt_all);
                const int i0 = ip * 2 * BM + static_cast<int>(cr) * BM;
                for (int kb = vg_first_kb<M>(ip); kb < nk && ok; ++kb) {
                    if (!mbar_wait(&b_empty[bs], ((bpar >> bs) & 1u) ^ 1u, limit)) {
                        raise_error(p.err, kErrTimeout, 17);
                        ok = false;
                        break;
                    }
                    if (cr == 0)
                        mbar_arrive_expect_tx(&b_full[bs], 2 * B_BYTES);
                    tma_load_2d_pair(b_base + bs * B_BYTES, &bmap, cluster_addr(&b_full[bs], 0), 0,
                                     (rt_all * nk + kb) * NCOLS + static_cast<int>(cr) * HALF);
                    bpar ^= 1u << bs;
                    bused |= 1u << bs;
                    bs = (bs + 1 == B_STAGES) ? 0 : bs + 1;
                    for (int pc = 0; pc < S::PIECES; ++pc) {
                        if (!mbar_wait(&a_empty[slot], ((apar >> slot) & 1u) ^ 1u, limit)) {
                            raise_error(p.err, kErrTimeout, 11);
                            ok = false;
                            break;
                        }
                        if (cr == 0)
                            mbar_arrive_expect_tx(&a_full[slot], 2 * A_TILE);
                        tma_load_3d_pair(a_base + slot * A_TILE, &fmap, cluster_addr(&a_full[slot], 0),
                                         kb * BK, i0, g * S::PIECES + pc);
                        apar ^= 1u << slot;
                        aused |= 1u << slot;
                        slot = (slot + 1 == NSLOT) ? 0 : slot + 1;
                    }
                }
            }
            if (!ok) {
                // let this CTA's copies land before the pair exits: the even CTA waits for the last
                // phase of each slot it armed; the odd CTA's copies are counted there, so it waits
                // a fixed time
                if (cr == 0) {
                    for (int s = 0; s < NSLOT; ++s)
                        if ((aused >> s) & 1u)
                            mbar_wait(&a_full[s], ((apar >> s) & 1u) ^ 1u, kPairDrainLimit);
                    for (int s = 0; s < B_STAGES; ++s)
                        if ((bused >> s) & 1u)
                            mbar_wait(&b_full[s], ((bpar >> s) & 1u) ^ 1u, kPairDrainLimit);
                } else {
                    const long long t0 = clock64();
                    while (clock64() - t0 < kPairDrainLimit) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue (even CTA)
        // Per K block: wait for both CTAs' right-operand halves, then for each piece of F wait for
        // both CTAs' tiles, issue four K=16 MMAs (M = 256 over the pair) and release the slot in
        // both CTAs; release the stage after the block, the accumulator after the segment.
        //   class-binned: H1 and H2 against all 256 columns; the first MMA after the diagonal pair
        //     block (K block 4 of the tile) halves what the accumulator holds.
        //   residual: H1 against all 256 columns, H2 against the R1 halves (N = 128) into the
        //     columns 64 .. 191, which belong to the same rows.
        if (cr == 0 && lane == 0) {
            int slot = 0, bstage = 0;
            uint32_t aph = 0u, bph = 0u;  // phase parity per slot / stage
            bool ok = true;
            int itn = 0;  // segments issued: accumulator itn % SETS
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, ip, rt_all;
                int64_t row0, row_end;
                vg_tile_coords<M>(p, tile, g, row0, row_end, ip, rt_all);
                const int klo = vg_first_kb<M>(ip);
                const int segk = S::SEGK > 0 ? S::SEGK : nk - klo;
                int acc = 0;
                for (int kb = klo; kb < nk && ok; ++kb) {
                    const int kr = kb - klo;
                    const bool seg_start = kr % segk == 0;
                    if (seg_start) {
                        acc = itn % S::SETS;
                        if (!mbar_wait_cluster(&tempty[acc], ((itn / S::SETS) & 1) ^ 1, limit)) {
                            raise_error(p.err, kErrTimeout, 13);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    if (!mbar_wait(&b_full[bstage], (bph >> bstage) & 1u, limit)) {
                        raise_error(p.err, kErrTimeout, 14);
                        ok = false;
                        break;
                    }
                    bph ^= 1u << bstage;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NCOLS);
                    const uint32_t sb = smem_u32(b_base + bstage * B_BYTES);
                    for (int pc = 0; pc < S::PIECES; ++pc) {
                        if (!mbar_wait(&a_full[slot], (aph >> slot) & 1u, limit)) {
                            raise_error(p.err, kErrTimeout, 16);
                            ok = false;
                            break;
                        }
                        aph ^= 1u << slot;
                        tc_fence_after();
                        const uint32_t sa = smem_u32(a_base + slot * A_TILE);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            // K-major, 128-byte swizzle: 16 k = 32 bytes along the row
                            const uint64_t ad = umma_desc_sw128(sa + kk * 32, 16, 1024);
                            const uint64_t bd = umma_desc_sw128(sb + kk * 32, 16, 1024);
                            const bool first = seg_start && pc == 0 && kk == 0;
                            if constexpr (M > 0) {
                                if (kr == PAIR_KB && pc == 0 && kk == 0)
                                    umma_f16_pair_halve_d(d_tmem, ad, bd, IDESC);
                                else
                                    umma_f16_pair(d_tmem, ad, bd, IDESC, first ? 0u : 1u);
                            } else {
                                if (pc == 0)
                                    umma_f16_pair(d_tmem, ad, bd, IDESC, first ? 0u : 1u);
                                else
                                    umma_f16_pair(d_tmem + NCOLS / 4, ad, bd, IDESC_R1, 1u);
                            }
                        }
                        umma_commit_pair(&a_empty[slot], PAIR);
                        slot = (slot + 1 == NSLOT) ? 0 : slot + 1;
                    }
                    if (!ok)
                        break;
                    umma_commit_pair(&b_empty[bstage], PAIR);
                    bstage = (bstage + 1 == B_STAGES) ? 0 : bstage + 1;
                    if (kr % segk == segk - 1 || kb + 1 == nk) {
                        umma_commit_pair(&tfull[acc], PAIR);
                        ++itn;
                    }
                }
            }
            umma_commit_pair(drain, 0x1);
            mbar_wait(drain, 0, kDrainLimit);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        // This CTA's TMEM: lane = one of its 128 coordinates, columns = all of the tile's columns.
        const int quarter = warp & 3;
        const int tid = quarter * 32 + lane;   // coordinate of this thread within the CTA's 128
        uint32_t tempty_leader[S::SETS];
#pragma unroll
        for (int a = 0; a < S::SETS; ++a)
            tempty_leader[a] = cluster_addr(&tempty[a], 0);
        int itn = 0;  // segments read: accumulator itn % SETS
        bool ok = true;
        auto wait_acc = [&](int acc) -> bool {
            int okw = 0;
            if (lane == 0)
                okw = mbar_wait(&tfull[acc], (itn / S::SETS) & 1, limit) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) {
                if (lane == 0)
                    raise_error(p.err, kErrTimeout, 15);
                return false;
            }
            __syncwarp();
            tc_fence_after();
            return true;
        };
        if constexpr (M > 0) {
            // Class binning. Per 32-column chunk (32 / M rows of M columns) all 128 threads stage
            // their coordinate's values in shared memory, then thread (pair pidx = row-in-chunk x
            // class q, part h) adds the values of the coordinates 4 ii + h (ii = 0..31) that have
            // class q, and the four parts combine in a fixed order: S[q][.] of the row.
            float *vs = reinterpret_cast<float *>(e_base);                 // [2][BM][VS_LD]
            uint8_t *qs = e_base + 2 * VS_BYTES;                           // [RT][BM] codes
            const int h = lane >> 3;
            const int pidx = (lane & 7) | (quarter << 3);
            const int rin = pidx / M, qcls = pidx % M;
            constexpr int ROWS_PER_CHUNK = 32 / M;
            const bool qvec = (p.d & 15) == 0 && (reinterpret_cast<uintptr_t>(p.Q) & 15u) == 0;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, ip, rt_all;
                int64_t row0, row_end;
                vg_tile_coords<M>(p, tile, g, row0, row_end, ip, rt_all);
                const int64_t ibase = static_cast<int64_t>(ip) * 2 * BM + static_cast<int64_t>(cr) * BM;
                const int ih = 2 * ip + static_cast<int>(cr);
                const bool halve_here = nk - vg_first_kb<M>(ip) <= PAIR_KB;  // no later block
                const int acc = itn % S::SETS;
                // All four warps take one verdict on the accumulator (so that none of them waits at
                // a named barrier the others have left); the barrier also ends the previous tile's
                // binning, so its codes may be overwritten.
                int okw = 0;
                if (lane == 0)
                    okw = mbar_wait(&tfull[acc], (itn / S::SETS) & 1, limit) ? 1 : 0;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!named_bar_and(EPI_BAR, EPI_THREADS, okw)) {
                    if (tid == 0)
                        raise_error(p.err, kErrTimeout, 15);
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the tile's codes at this CTA's coordinates (0xFF: no coordinate or no row)
                for (int e = tid; e < S::RT * (BM / 16); e += EPI_THREADS) {
                    const int r = e / (BM / 16), c16 = e % (BM / 16);
                    const int64_t j = row0 + r, k = ibase + 16 * c16;
                    uint4 qv = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
                    if (j < row_end && k < p.d) {
                        if (qvec && k + 16 <= p.d) {
                            qv = *reinterpret_cast<const uint4 *>(p.Q + j * p.d + k);
                        } else {
                            uint8_t *b = reinterpret_cast<uint8_t *>(&qv);
                            for (int e2 = 0; e2 < 16; ++e2)
                                if (k + e2 < p.d)
                                    b[e2] = p.Q[j * p.d + k + e2];
                        }
                    }
                    *reinterpret_cast<uint4 *>(qs + r * BM + 16 * c16) = qv;
                }
                const int64_t i = ibase + tid;
                // the accumulator carries 2^fexp[i]; tiles without a block after the diagonal one
                // are halved here
                const float inv_si = pow2f(i < p.d ? -p.fexp[static_cast<int64_t>(g) * p.d + i] : 0) *
                                     (halve_here ? 0.5f : 1.f);
#pragma unroll 1
                for (int ch = 0; ch < NCOLS / 32; ++ch) {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                           static_cast<uint32_t>(acc * NCOLS + ch * 32),
                                       v);
                    if (ch + 1 == NCOLS / 32) {
                        tc_fence_before();
                        mbar_arrive_cluster(tempty_leader[acc]);   // the accumulator is free
                    }
                    float *vrow = vs + (ch & 1) * (BM * VS_LD) + tid * VS_LD;
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        *reinterpret_cast<float4 *>(vrow + 4 * e4) =
                            make_float4(v[4 * e4] * inv_si, v[4 * e4 + 1] * inv_si,
                                        v[4 * e4 + 2] * inv_si, v[4 * e4 + 3] * inv_si);
                    named_bar_sync(EPI_BAR, EPI_THREADS);      // the chunk (and the codes) staged
                    const int rr = ch * ROWS_PER_CHUNK + rin;  // row of the tile
                    const float *vcol = vs + (ch & 1) * (BM * VS_LD) + rin * M;
                    const uint8_t *qrow = qs + rr * BM;
                    float sacc[M];
#pragma unroll
                    for (int c = 0; c < M; ++c)
                        sacc[c] = 0.f;
#pragma unroll 8
                    for (int ii = 0; ii < BM / 4; ++ii) {
                        const int il = 4 * ii + h;
                        const bool mine = qrow[il] == qcls;
                        const float *vv = vcol + il * VS_LD;
                        if constexpr (M >= 4) {
#pragma unroll
                            for (int c4 = 0; c4 < M / 4; ++c4) {
                                const float4 x = *reinterpret_cast<const float4 *>(vv + 4 * c4);
                                if (mine) {
                                    sacc[4 * c4] += x.x;
                                    sacc[4 * c4 + 1] += x.y;
                                    sacc[4 * c4 + 2] += x.z;
                                    sacc[4 * c4 + 3] += x.w;
                                }
                            }
                        } else {
                            const float2 x = *reinterpret_cast<const float2 *>(vv);
                            if (mine) {
                                sacc[0] += x.x;
                                sacc[1] += x.y;
                            }
                        }
                    }
                    // parts h and h ^ 1, then the two pairs: the same order on every lane
#pragma unroll
                    for (int c = 0; c < M; ++c) {
                        sacc[c] += __shfl_xor_sync(0xffffffffu, sacc[c], 8);
                        sacc[c] += __shfl_xor_sync(0xffffffffu, sacc[c], 16);
                    }
                    const int64_t j = row0 + rr;
                    if (h == 0 && j < row_end) {
                        float *dst = p.S + ((static_cast<int64_t>(ih) * p.d_out + j) * M + qcls) * M;
                        if constexpr (M >= 4) {
#pragma unroll
                            for (int c4 = 0; c4 < M / 4; ++c4)
                                reinterpret_cast<float4 *>(dst)[c4] =
                                    make_float4(sacc[4 * c4], sacc[4 * c4 + 1], sacc[4 * c4 + 2],
                                                sacc[4 * c4 + 3]);
                        } else {
                            *reinterpret_cast<float2 *>(dst) = make_float2(sacc[0], sacc[1]);
                        }
                    }
                }
                ++itn;
            }
        } else {
            // Residual sums: per segment, each of the tile's 128 rows adds its columns (R1 column,
            // and the R2 column that also holds H2 x R1) into an fp32 sum held in registers.
            const int nseg = (nk + S::SEGK - 1) / S::SEGK;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, ip, rt_all;
                int64_t row0, row_end;
                vg_tile_coords<M>(p, tile, g, row0, row_end, ip, rt_all);
                const int64_t i = static_cast<int64_t>(ip) * 2 * BM + static_cast<int64_t>(cr) * BM + tid;
                const float inv_si = pow2f(i < p.d ? -p.fexp[static_cast<int64_t>(g) * p.d + i] : 0);
                float uacc[S::RT];
#pragma unroll
                for (int r = 0; r < S::RT; ++r)
                    uacc[r] = 0.f;
                for (int sg = 0; sg < nseg; ++sg, ++itn) {
                    const int acc = itn % S::SETS;
                    if (!wait_acc(acc)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int ch = 0; ch < NCOLS / 32; ++ch) {
                        float v[32];
                        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                               static_cast<uint32_t>(acc * NCOLS + ch * 32),
                                           v);
                        // column c belongs to row (c / 128) * 64 + c % 64
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = ch * 32 + e;
                            uacc[(col >> 7) * 64 + (col & 63)] += v[e];
                        }
                        // the chunk's sums are complete here, before the next chunk is loaded
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = ch * 32 + e;
                            asm volatile("" : "+f"(uacc[(col >> 7) * 64 + (col & 63)]));
                        }
                    }
                    tc_fence_before();
                    mbar_arrive_cluster(tempty_leader[acc]);
                }
                if (!ok)
                    break;
                if (i < p.d) {
#pragma unroll
                    for (int r = 0; r < S::RT; ++r) {
                        const int64_t j = row0 + r;
                        if (j < row_end)
                            p.U[j * p.d + i] = (uacc[r] * inv_si) * pow2f(-p.rexp[j]);
                    }
                }
            }
        }
    }

    // Both CTAs stay until the pair is done: the MMAs read both CTAs' shared memory and the
    // copies and epilogues of both signal barriers in the even CTA.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
cudaError_t lnq_split_f16(const float *F, int64_t d, int groups, __half *Fh, int32_t *fexp,
                          cudaStream_t s)
{
    KernelTimer timer("lnq_split_f16", s);
    split_f16_kernel<<<static_cast<unsigned>(d * groups), 256, 0, s>>>(F, d, Fh, fexp);
    return cudaGetLastError();
}

cudaError_t lnq_residual_scale(const uint8_t *Q, const float *W, const float *C, int64_t d,
                               int64_t d_out, int m, int32_t *rexp, cudaStream_t s)
{
    KernelTimer timer("lnq_residual_scale", s);
    residual_scale_kernel<<<static_cast<unsigned>((d_out + 7) / 8), 256, 0, s>>>(Q, W, C, d, d_out,
                                                                                m, rexp);
    return cudaGetLastError();
}

// Tensor map over F's pieces [groups * planes][d][ld] (two fp16 planes per group):
// 64 x 128 (column x row) boxes, 128-byte swizzle; reads outside d x d return zeros.
static bool encode_pieces_map(CUtensorMap *map, const void *pieces, int64_t d, int planes,
                              CUtensorMapDataType type)
{
    auto encode = tensor_map_encoder();
    if (encode == nullptr)
        return false;
    const int64_t ld = pieces_stride(d);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(d),
                          static_cast<cuuint64_t>(planes)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(d * ld) * 2};
    cuuint32_t box[3] = {vg::BK, vg::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, type, 3, const_cast<void *>(pieces), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over the fp16 pieces Fh [groups][2][d][ld].
bool encode_f16_pieces(CUtensorMap *map, const __half *Fh, int64_t d, int groups)
{
    return encode_pieces_map(map, Fh, d, groups * 2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

// Right-operand image rows for m (M > 0 layout) or for the residual product: the workspace holds
// the larger of the two.
template <int M>
static int64_t image_rows_m(int64_t d, int64_t d_out, int groups)
{
    using S = VgShape<M>;
    const int64_t R = d_out / groups;
    const int64_t nk = (d + vg::BK - 1) / vg::BK;
    return groups * ((R + S::RT - 1) / S::RT) * nk * vg::NCOLS;
}

size_t lnq_vgemm_image_bytes(int64_t d, int64_t d_out, int groups, int m)
{
    int64_t rows = image_rows_m<0>(d, d_out, groups);
    int64_t rm = 0;
    switch (m) {
    case 2: rm = image_rows_m<2>(d, d_out, groups); break;
    case 4: rm = image_rows_m<4>(d, d_out, groups); break;
    case 8: rm = image_rows_m<8>(d, d_out, groups); break;
    case 16: rm = image_rows_m<16>(d, d_out, groups); break;
    }
    if (rm > rows)
        rows = rm;
    return static_cast<size_t>(rows) * 64 * 2;
}

// Class-binned partial sums: one m x m block per row and per 128 coordinates.
size_t lnq_binned_bytes(int64_t d, int64_t d_out, int m)
{
    const int64_t halves = 2 * ((d + 2 * vg::BM - 1) / (2 * vg::BM));
    return static_cast<size_t>(halves) * d_out * m * m * sizeof(float);
}

template <int M>
static cudaError_t launch_vgemm_m(const CUtensorMap &map, VgParams p, const float *W,
                                  const float *C, int m, uint16_t *img, int num_sms,
                                  cudaStream_t s, const char *name)
{
    using S = VgShape<M>;
    p.row_tiles_per_group = static_cast<int>((p.rows_per_group + S::RT - 1) / S::RT);
    p.i_pairs = static_cast<int>((p.d + 2 * vg::BM - 1) / (2 * vg::BM));
    const int64_t groups = p.d_out / p.rows_per_group;
    const int nk = static_cast<int>((p.d + vg::BK - 1) / vg::BK);
    const int64_t num_rt_all = groups * p.row_tiles_per_group;
    const int64_t img_rows = num_rt_all * nk * vg::NCOLS;
    if (img_rows > 0x7fffffffLL || num_rt_all * p.i_pairs > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    p.num_tiles = static_cast<int>(num_rt_all * p.i_pairs);
    {
        KernelTimer timer(M > 0 ? "lnq_operand_image" : "lnq_residual_image", s);
        // one task per (row tile, row, 8 coordinates)
        const int64_t ntasks = num_rt_all * nk * S::RT * 8;
        int64_t tblocks = (ntasks + 255) / 256;
        if (tblocks > static_cast<int64_t>(num_sms) * 16)
            tblocks = static_cast<int64_t>(num_sms) * 16;
        if constexpr (M > 0) {
            onehot_image_kernel<M><<<static_cast<unsigned>(tblocks), 256, 0, s>>>(
                p.Q, p.d, p.rows_per_group, p.row_tiles_per_group, ntasks, nk, img);
        } else {
            residual_image_kernel<<<static_cast<unsigned>(tblocks), 256, 0, s>>>(
                p.Q, W, C, p.rexp, p.d, p.rows_per_group, p.row_tiles_per_group, ntasks, nk, m,
                img);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    CUtensorMap bmap;
    {
        auto encode = tensor_map_encoder();
        if (encode == nullptr)
            return cudaErrorInvalidValue;
        cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(img_rows)};
        cuuint64_t strides[1] = {128};
        cuuint32_t box[2] = {64, static_cast<cuuint32_t>(vg::HALF)};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&bmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, img, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(lnq_vgemm_kernel<M>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(S::SMEM));
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(vg::NUM_THREADS);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once (at most one CTA per SM)
    static int resident[5] = {0, 0, 0, 0, 0};
    constexpr int slot = M == 0 ? 0 : (M == 2 ? 1 : (M == 4 ? 2 : (M == 8 ? 3 : 4)));
    if (resident[slot] == 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, lnq_vgemm_kernel<M>, &cfg) != cudaSuccess ||
            clusters < 1) {
            (void)cudaGetLastError();   // a failed query is not an error of this call
            clusters = num_sms / 2;
        }
        resident[slot] = clusters;
    }
    int pairs = resident[slot];
    if (pairs > p.num_tiles)
        pairs = p.num_tiles;
    if (pairs < 1)
        pairs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    KernelTimer timer(name, s);
    e = cudaLaunchKernelEx(&cfg, lnq_vgemm_kernel<M>, map, bmap, p);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

// The class-binned partial sums Sb of M = P^T F P for every row (m in {2,4,8,16}), or, with
// residual_only, U = F r with the residual scales rexp (C == nullptr: the zero codebook, U = -F w),
// both from the fp16 pieces (Fh, fexp).
cudaError_t lnq_vgemm(const __half *Fh, const int32_t *fexp, const int32_t *rexp, int groups,
                      const uint8_t *Q, const float *W, const float *C, float *Sb, float *U,
                      uint16_t *img, int64_t d, int64_t d_out, int m, bool residual_only,
                      DeviceErr err, int num_sms, cudaStream_t s)
{
    CUtensorMap map;
    if (!encode_f16_pieces(&map, Fh, d, groups))
        return cudaErrorInvalidValue;
    VgParams p{};
    p.Q = Q;
    p.S = Sb;
    p.U = U;
    p.fexp = fexp;
    p.rexp = rexp;
    p.d = d;
    p.d_out = d_out;
    p.rows_per_group = d_out / groups;
    p.err = err;
    if (residual_only)
        return launch_vgemm_m<0>(map, p, W, C, m, img, num_sms, s, "lnq_residual_gemm");
    switch (m) {
    case 2: return launch_vgemm_m<2>(map, p, W, C, m, img, num_sms, s, "lnq_mgemm");
    case 4: return launch_vgemm_m<4>(map, p, W, C, m, img, num_sms, s, "lnq_mgemm");
    case 8: return launch_vgemm_m<8>(map, p, W, C, m, img, num_sms, s, "lnq_mgemm");
    case 16: return launch_vgemm_m<16>(map, p, W, C, m, img, num_sms, s, "lnq_mgemm");
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
