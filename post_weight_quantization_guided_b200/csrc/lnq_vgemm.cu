// lnq_vgemm.cu -- the dense contraction of an LNQ iteration on tcgen05 tensor cores.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section. The codebook update
// c <- (P^T F P)^-1 P^T F w needs, per output row j, the class-binned products V_j = F P_j
// (d x m; P_j is the one-hot assignment) and the residual gradient u_j = F r_j with
// r_j = c_j[q_j] - w_j. For all rows of one Fisher group these are a single product
//
//      [V_j1 | u_j1 | V_j2 | u_j2 | ...] = F x [P_j1 | r_j1 | P_j2 | r_j2 | ...]
//
// whose left operand F is shared by every row of the group. This kernel computes it with
// tcgen05.mma.kind::f16, exactly in fp32 terms:
//   * F (fp32) is split into three bf16 pieces F = F1 + F2 + F3 (exact for normal values), and
//     the three products accumulate into one TMEM accumulator;
//   * the one-hot columns are 0/1 (exact in bf16); r is split the same way into three bf16
//     pieces, one column each, so u = sum of nine exact bf16 x bf16 products;
//   * accumulation is fp32 in TMEM.
// A tile is 128 coordinates (i) x 256 columns (RT rows x (m one-hot + 3 residual pieces), RT =
// floor(256 / (m + 3))). F tiles arrive by TMA (K-major, 128-byte swizzle); the 256 x 64 right
// operand tile is generated in shared memory from Q, C and W by four producer warps, in the
// same swizzled K-major layout. The epilogue writes V[j][i][b] and uT[i][j] (u transposed, so
// the sweep reads it coalesced). With m = 0 the kernel computes u = F r only (85 rows per tile),
// which the objective uses.
#include <cuda_bf16.h>

#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

namespace vg {
constexpr int BM = 128;
constexpr int BK = 64;
constexpr int PIECES = 3;
constexpr int A_TILE = BM * BK * 2;              // one bf16 piece of a 128 x 64 F tile: 16 KB
constexpr int B_STAGES = 2;
constexpr int NUM_THREADS = 320;                 // w0 TMA, w1 MMA, w2-5 epilogue, w6-9 operand
constexpr int PRODUCER_THREADS = 128;
constexpr int TMEM_COLS = 512;
constexpr int MAX_DYN_SMEM = 232448;             // opt-in dynamic shared memory per block
constexpr int BAR_BYTES = 512;
}  // namespace vg

// Tile shapes. With one-hot columns (M > 0) a tile is 256 columns and two TMEM accumulators
// alternate between tiles. The residual-only product (M == 0) feeds the objective, which sums
// r_i u_i with cancellation; there a tile is 128 columns and the K range is cut into four
// segments with one accumulator each, so each fp32 accumulator takes a quarter of the additions.
// Shared memory: A arrives one bf16 piece (16 KB) per slot, in as many slots as fit next to the two
// right-operand stages and the staging area, so that several K blocks of F are in flight.
template <int M>
struct VgShape {
    static constexpr int NCOLS = M > 0 ? 256 : 128;     // MMA N
    static constexpr int SEGS = M > 0 ? 1 : 4;          // K segments (one accumulator each)
    static constexpr int SETS = M > 0 ? 2 : 1;          // accumulator sets (tile double-buffer)
    static constexpr int RT = NCOLS / (M + 3);          // rows per tile
    static constexpr int ONEHOT = RT * M;               // one-hot columns
    static constexpr int USED = RT * (M + 3);           // columns carrying data
    static constexpr int CHUNKS = (USED + 31) / 32;     // 32-column TMEM loads per accumulator
    static constexpr int B_BYTES = NCOLS * 128;         // N rows x 64 k of bf16
    static constexpr int STG_BYTES = RT * 512;          // staging: classes, residual pieces, codebook
    static constexpr int A_FIT = (vg::MAX_DYN_SMEM - 1024 - vg::BAR_BYTES -
                                  vg::B_STAGES * B_BYTES - STG_BYTES) / vg::A_TILE;
    static constexpr int A_SLOTS = A_FIT < 12 ? A_FIT : 12;
    static constexpr size_t SMEM = 1024 + static_cast<size_t>(A_SLOTS) * vg::A_TILE +
                                   vg::B_STAGES * B_BYTES + vg::BAR_BYTES + STG_BYTES;
    static_assert(SETS * SEGS * NCOLS <= vg::TMEM_COLS, "TMEM holds 512 fp32 columns");
    static_assert(A_SLOTS >= 2 * vg::PIECES, "at least two K blocks of F in flight");
    static_assert(SMEM <= vg::MAX_DYN_SMEM, "shared memory");
};

__device__ __forceinline__ uint16_t bf16_bits(float x)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// The three bf16 pieces of x: x == p0 + p1 + p2 exactly for normal fp32 x.
__device__ __forceinline__ void split3(float x, float &p0, float &p1, float &p2)
{
    p0 = __bfloat162float(__float2bfloat16_rn(x));
    const float r1 = x - p0;
    p1 = __bfloat162float(__float2bfloat16_rn(r1));
    p2 = r1 - p1;
}

// Row stride (elements) of the bf16 pieces: TMA needs row strides that are multiples of 16 B.
__host__ __device__ inline int64_t pieces_stride(int64_t d) { return (d + 7) / 8 * 8; }

// F (fp32 [groups][d][d]) -> Fp (bf16 [groups][3][d][ld]), ld = pieces_stride(d), zero padded.
__global__ void split_f_kernel(const float *__restrict__ F, int64_t d, int groups,
                               __nv_bfloat16 *__restrict__ Fp)
{
    const int64_t ld = pieces_stride(d);
    const int64_t plane = d * ld;
    const int64_t total = plane * groups;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t g = e / plane, r = e - g * plane;
        const int64_t row = r / ld, col = r - row * ld;
        float p0 = 0.f, p1 = 0.f, p2 = 0.f;
        if (col < d)
            split3(F[(g * d + row) * d + col], p0, p1, p2);
        __nv_bfloat16 *base = Fp + g * 3 * plane + r;
        base[0] = __float2bfloat16_rn(p0);
        base[plane] = __float2bfloat16_rn(p1);
        base[2 * plane] = __float2bfloat16_rn(p2);
    }
}

struct VgParams {
    const uint8_t *Q;   // [d_out][d]
    const float *W;     // [d_out][d]
    const float *C;     // [d_out][m]
    float *V;           // [d_out][d][m] (m > 0)
    float *uT;          // [d][d_out]
    int64_t d, d_out, rows_per_group;
    int m;
    int row_tiles_per_group, i_tiles, num_tiles;
    DeviceErr err;
};

template <int M>
__device__ __forceinline__ void vg_tile_coords(const VgParams &p, int tile, int &g, int64_t &row0,
                                               int64_t &row_end, int &it)
{
    constexpr int RT = VgShape<M>::RT;
    it = tile % p.i_tiles;
    const int rt_all = tile / p.i_tiles;
    g = rt_all / p.row_tiles_per_group;
    const int rt = rt_all - g * p.row_tiles_per_group;
    const int64_t gstart = static_cast<int64_t>(g) * p.rows_per_group;
    row0 = gstart + static_cast<int64_t>(rt) * RT;
    row_end = min(row0 + RT, gstart + p.rows_per_group);
}

// Per-K-block staging of the right operand's sources, shared by the producer warps:
//   q[r][kk]     class of coordinate k0+kk in row row0+r (0xFF outside the problem)
//   rp[r][p][kk] bf16 piece p of the residual c[q] - w of that coordinate (0 outside)
//   c[r][b]      codebook of row row0+r
template <int RT>
struct VgStage {
    uint8_t q[RT][64];
    uint16_t rp[RT][3][64];
    float c[RT][16];
};

template <int M>
__global__ void __launch_bounds__(vg::NUM_THREADS, 1)
    lnq_vgemm_kernel(const __grid_constant__ CUtensorMap fmap, VgParams p)
{
    using namespace vg;
    using S = VgShape<M>;
    constexpr int NSLOT = S::A_SLOTS;
    constexpr uint32_t IDESC = umma_idesc_f16kind(BM, S::NCOLS, false, false, /*f16=*/false);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t *a_base = smem;                                       // [NSLOT][16 KB]
    uint8_t *b_base = smem + NSLOT * A_TILE;                      // [B_STAGES][B_BYTES]
    uint64_t *bars = reinterpret_cast<uint64_t *>(b_base + B_STAGES * S::B_BYTES);
    uint64_t *a_full = bars;                                      // [NSLOT]
    uint64_t *a_empty = a_full + NSLOT;                           // [NSLOT]
    uint64_t *b_full = a_empty + NSLOT;                           // [B_STAGES]
    uint64_t *b_empty = b_full + B_STAGES;                        // [B_STAGES]
    uint64_t *tfull = b_empty + B_STAGES;                         // [SETS]
    uint64_t *tempty = tfull + S::SETS;                           // [SETS]
    uint64_t *drain = tempty + S::SETS;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    VgStage<S::RT> &stg = *reinterpret_cast<VgStage<S::RT> *>(
        b_base + B_STAGES * S::B_BYTES + BAR_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&b_full[s], PRODUCER_THREADS);
            mbar_init(&b_empty[s], 1);
        }
        for (int a = 0; a < S::SETS; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4 * 32);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&fmap);
    }
    if (warp == 1)
        tmem_alloc(tmem_holder, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int nk = static_cast<int>((p.d + BK - 1) / BK);
    const long long limit = p.err.limit;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA: F pieces
        // One 16 KB piece tile per slot, slots in round-robin order.
        if (lane == 0) {
            int fills[NSLOT] = {};
            int slot = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                int g, it;
                int64_t row0, row_end;
                vg_tile_coords<M>(p, tile, g, row0, row_end, it);
                for (int kb = 0; kb < nk && ok; ++kb) {
                    for (int pc = 0; pc < PIECES; ++pc) {
                        if (!mbar_wait(&a_empty[slot], (fills[slot] & 1) ^ 1, limit)) {
                            raise_error(p.err, kErrTimeout, 11);
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&a_full[slot], A_TILE);
                        tma_load_3d(a_base + slot * A_TILE, &fmap, &a_full[slot], kb * BK, it * BM,
                                    g * PIECES + pc);
                        ++fills[slot];
                        slot = (slot + 1 == NSLOT) ? 0 : slot + 1;
                    }
                }
            }
            if (!ok)
                for (int s = 0; s < NSLOT; ++s)
                    if (fills[s] > 0)
                        mbar_wait(&a_full[s], (fills[s] - 1) & 1, kDrainLimit);
        }
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- right operand
        // Four warps build the right operand of each K block in two phases, separated by a named
        // barrier. Staging: each thread takes quads of 4 consecutive k of one row (prefetched into
        // registers during the previous block) and writes the classes and the three bf16 pieces of
        // the residuals. Expansion: each thread takes one (row, 16-byte column chunk): it reads the
        // 8 classes once and writes the chunk of every one-hot row of that row, then copies residual
        // chunks. Loads are issued before stores so that shared-memory accesses overlap. The stage
        // wait is ANDed over the four warps, so they leave together on a timeout and the named
        // barriers cannot deadlock. Columns beyond S::USED are never written: the epilogue ignores
        // them.
        constexpr int kBar = 1;
        constexpr int QUADS = S::RT * 16;
        constexpr int PER = (QUADS + PRODUCER_THREADS - 1) / PRODUCER_THREADS;
        constexpr int PAIRS = S::RT * 8;
        constexpr int RCH = 3 * S::RT * 8;  // residual chunks
        constexpr int RPER = (RCH + PRODUCER_THREADS - 1) / PRODUCER_THREADS;
        const int t = threadIdx.x - 6 * 32;
        const bool vec = (p.d & 3) == 0 && (reinterpret_cast<uintptr_t>(p.Q) & 3u) == 0 &&
                         (reinterpret_cast<uintptr_t>(p.W) & 15u) == 0;
        int uses[B_STAGES] = {};
        int stage = 0;
        bool ok = true;
        uint32_t qpre[PER];
        float4 wpre[PER];
        auto fetch = [&](int64_t row0, int64_t row_end, int64_t k0) {
#pragma unroll
            for (int s2 = 0; s2 < PER; ++s2) {
                const int e = t + s2 * PRODUCER_THREADS;
                const int r = e >> 4, kk = (e & 15) * 4;
                const int64_t j = row0 + r, k = k0 + kk;
                qpre[s2] = 0xFFFFFFFFu;
                wpre[s2] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < QUADS && j < row_end && k < p.d) {
                    if (vec) {
                        qpre[s2] = *reinterpret_cast<const uint32_t *>(p.Q + j * p.d + k);
                        wpre[s2] = *reinterpret_cast<const float4 *>(p.W + j * p.d + k);
                    } else {
                        uint32_t qv = 0;
                        float wv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const bool in = k + e4 < p.d;
                            qv |= static_cast<uint32_t>(in ? p.Q[j * p.d + k + e4] : 0xFFu) << (8 * e4);
                            wv[e4] = in ? p.W[j * p.d + k + e4] : 0.f;
                        }
                        qpre[s2] = qv;
                        wpre[s2] = make_float4(wv[0], wv[1], wv[2], wv[3]);
                    }
                }
            }
        };
        for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
            int g, it;
            int64_t row0, row_end;
            vg_tile_coords<M>(p, tile, g, row0, row_end, it);
            fetch(row0, row_end, 0);
            for (int kb = 0; kb < nk; ++kb) {
                const int mine = mbar_wait(&b_empty[stage], (uses[stage] & 1) ^ 1, limit) ? 1 : 0;
                if (!named_bar_and(kBar, PRODUCER_THREADS, mine)) {
                    if (t == 0)
                        raise_error(p.err, kErrTimeout, 12);
                    ok = false;
                    break;
                }
                if (kb == 0) {
                    for (int e = t; e < S::RT * 16; e += PRODUCER_THREADS) {
                        const int r = e >> 4, b = e & 15;
                        const int64_t j = row0 + r;
                        stg.c[r][b] = (j < row_end && b < p.m) ? p.C[j * p.m + b] : 0.f;
                    }
                    named_bar_sync(kBar, PRODUCER_THREADS);
                }
                // staging: classes and residual pieces of this K block
                float cq[PER][4];
#pragma unroll
                for (int s2 = 0; s2 < PER; ++s2) {
                    const int e = t + s2 * PRODUCER_THREADS;
                    const int r = (e < QUADS) ? (e >> 4) : 0;
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const uint32_t qv = (qpre[s2] >> (8 * e4)) & 0xFFu;
                        cq[s2][e4] = stg.c[r][(qv == 0xFFu ? 0u : qv) & (p.m - 1)];
                    }
                }
#pragma unroll
                for (int s2 = 0; s2 < PER; ++s2) {
                    const int e = t + s2 * PRODUCER_THREADS;
                    if (e < QUADS) {
                        const int r = e >> 4, kk = (e & 15) * 4;
                        const float wv[4] = {wpre[s2].x, wpre[s2].y, wpre[s2].z, wpre[s2].w};
                        uint32_t pk[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
                        uint32_t qmask = 0u;
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const uint32_t qv = (qpre[s2] >> (8 * e4)) & 0xFFu;
                            float p0 = 0.f, p1 = 0.f, p2 = 0.f;
                            if (qv != 0xFFu) {
                                split3(cq[s2][e4] - wv[e4], p0, p1, p2);
                                qmask |= (qv & (p.m - 1)) << (8 * e4);
                            } else {
                                qmask |= 0xFFu << (8 * e4);
                            }
                            pk[0][e4 >> 1] |= static_cast<uint32_t>(bf16_bits(p0)) << (16 * (e4 & 1));
                            pk[1][e4 >> 1] |= static_cast<uint32_t>(bf16_bits(p1)) << (16 * (e4 & 1));
                            pk[2][e4 >> 1] |= static_cast<uint32_t>(bf16_bits(p2)) << (16 * (e4 & 1));
                        }
                        *reinterpret_cast<uint32_t *>(&stg.q[r][kk]) = qmask;
#pragma unroll
                        for (int pc = 0; pc < 3; ++pc)
                            *reinterpret_cast<uint2 *>(&stg.rp[r][pc][kk]) = make_uint2(pk[pc][0], pk[pc][1]);
                    }
                }
                if (kb + 1 < nk)
                    fetch(row0, row_end, static_cast<int64_t>(kb + 1) * BK);
                named_bar_sync(kBar, PRODUCER_THREADS);
                // expansion into the swizzled K-major tile
                uint8_t *sb = b_base + stage * S::B_BYTES;
                if constexpr (M > 0) {
                    for (int pi = t; pi < PAIRS; pi += PRODUCER_THREADS) {
                        const int r = pi >> 3, c = pi & 7;
                        const uint2 qq = *reinterpret_cast<const uint2 *>(&stg.q[r][8 * c]);
#pragma unroll
                        for (int b = 0; b < M; ++b) {
                            const int n = r * M + b;
                            const uint32_t bbbb = 0x01010101u * static_cast<uint32_t>(b);
                            const uint32_t m0 = __vcmpeq4(qq.x, bbbb), m1 = __vcmpeq4(qq.y, bbbb);
                            // byte e of the mask (0xFF or 0) -> bf16 1.0 (0x3F80) or 0, half-word e
                            *reinterpret_cast<uint4 *>(sb + n * 128 + ((c ^ (n & 7)) << 4)) =
                                make_uint4(__byte_perm(m0, 0u, 0x1100) & 0x3F803F80u,
                                           __byte_perm(m0, 0u, 0x3322) & 0x3F803F80u,
                                           __byte_perm(m1, 0u, 0x1100) & 0x3F803F80u,
                                           __byte_perm(m1, 0u, 0x3322) & 0x3F803F80u);
                        }
                    }
                }
                {
                    uint4 rv[RPER];
#pragma unroll
                    for (int s2 = 0; s2 < RPER; ++s2) {
                        const int ci = t + s2 * PRODUCER_THREADS;
                        const int nr = ci >> 3, c = ci & 7;   // nr = 3 r + piece
                        if (ci < RCH)
                            rv[s2] = *reinterpret_cast<const uint4 *>(&stg.rp[nr / 3][nr % 3][8 * c]);
                    }
#pragma unroll
                    for (int s2 = 0; s2 < RPER; ++s2) {
                        const int ci = t + s2 * PRODUCER_THREADS;
                        const int nr = ci >> 3, c = ci & 7;
                        const int n = S::ONEHOT + nr;
                        if (ci < RCH)
                            *reinterpret_cast<uint4 *>(sb + n * 128 + ((c ^ (n & 7)) << 4)) = rv[s2];
                    }
                }
                // make the generic-proxy writes visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(&b_full[stage]);
                ++uses[stage];
                stage = (stage + 1 == B_STAGES) ? 0 : stage + 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // Per K block: wait for the right operand, then for each piece wait for its A slot, issue
        // four K=16 MMAs and release the slot; release the right-operand stage after the block.
        if (lane == 0) {
            int bstage = 0, slot = 0;
            uint32_t bphase[B_STAGES] = {};
            uint32_t aphase[NSLOT] = {};
            bool ok = true;
            int itn = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++itn) {
                const int acc = itn % S::SETS;
                const int use = itn / S::SETS;
                if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, limit)) {
                    raise_error(p.err, kErrTimeout, 13);
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < nk && ok; ++kb) {
                    if (!mbar_wait(&b_full[bstage], bphase[bstage], limit)) {
                        raise_error(p.err, kErrTimeout, 14);
                        ok = false;
                        break;
                    }
                    bphase[bstage] ^= 1u;
                    const int seg = (kb * S::SEGS) / nk;
                    const bool seg_start = (kb == 0) || (((kb - 1) * S::SEGS) / nk != seg);
                    const uint32_t d_tmem =
                        tmem_base + static_cast<uint32_t>((acc * S::SEGS + seg) * S::NCOLS);
                    const uint32_t sb = smem_u32(b_base + bstage * S::B_BYTES);
                    for (int pc = 0; pc < PIECES; ++pc) {
                        if (!mbar_wait(&a_full[slot], aphase[slot], limit)) {
                            raise_error(p.err, kErrTimeout, 16);
                            ok = false;
                            break;
                        }
                        aphase[slot] ^= 1u;
                        tc_fence_after();
                        const uint32_t sa = smem_u32(a_base + slot * A_TILE);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            // K-major, 128-byte swizzle: 16 k = 32 bytes along the row.
                            const uint64_t ad = umma_desc_sw128(sa + kk * 32, 16, 1024);
                            const uint64_t bd = umma_desc_sw128(sb + kk * 32, 16, 1024);
                            umma_f16(d_tmem, ad, bd, IDESC,
                                     (!seg_start || pc != 0 || kk != 0) ? 1u : 0u);
                        }
                        umma_commit(&a_empty[slot]);
                        slot = (slot + 1 == NSLOT) ? 0 : slot + 1;
                    }
                    if (!ok)
                        break;
                    umma_commit(&b_empty[bstage]);
                    bstage = (bstage + 1 == B_STAGES) ? 0 : bstage + 1;
                }
                if (!ok)
                    break;
                umma_commit(&tfull[acc]);
            }
            umma_commit(drain);
            mbar_wait(drain, 0, kDrainLimit);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        const int quarter = warp & 3;
        int itn = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++itn) {
            const int acc = itn % S::SETS;
            const int use = itn / S::SETS;
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait(&tfull[acc], use & 1, limit) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0)
                    raise_error(p.err, kErrTimeout, 15);
                break;
            }
            __syncwarp();
            tc_fence_after();
            int g, it;
            int64_t row0, row_end;
            vg_tile_coords<M>(p, tile, g, row0, row_end, it);
            const int64_t i = static_cast<int64_t>(it) * BM + quarter * 32 + lane;
            float uacc[S::RT];
#pragma unroll
            for (int r = 0; r < S::RT; ++r)
                uacc[r] = 0.f;
            for (int seg = 0; seg < S::SEGS; ++seg) {
                // K block kb feeds segment kb * SEGS / nk; skip segments that received none
                const int first = (seg * nk + S::SEGS - 1) / S::SEGS;
                if (first >= nk || (first * S::SEGS) / nk != seg)
                    continue;
#pragma unroll
                for (int ch = 0; ch < S::CHUNKS; ++ch) {
                    float v[32];
                    const uint32_t taddr =
                        tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                        static_cast<uint32_t>((acc * S::SEGS + seg) * S::NCOLS + ch * 32);
                    tmem_ld_32x32b_x32(taddr, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int col = ch * 32 + e;
                        if constexpr (M > 0) {
                            // M divides 32, so each row's M columns sit inside one chunk.
                            if (col < S::ONEHOT && col % M == 0) {
                                const int64_t j = row0 + col / M;
                                if (j < row_end && i < p.d) {
                                    float *dst = p.V + (j * p.d + i) * M;
                                    if constexpr (M >= 4) {
#pragma unroll
                                        for (int b4 = 0; b4 < M / 4; ++b4)
                                            reinterpret_cast<float4 *>(dst)[b4] =
                                                make_float4(v[e + 4 * b4], v[e + 4 * b4 + 1],
                                                            v[e + 4 * b4 + 2], v[e + 4 * b4 + 3]);
                                    } else {
                                        *reinterpret_cast<float2 *>(dst) =
                                            make_float2(v[e], v[e + 1]);
                                    }
                                }
                            }
                        }
                        if (col >= S::ONEHOT && col < S::USED)
                            uacc[(col - S::ONEHOT) / 3] += v[e];
                    }
                }
            }
            if (i < p.d) {
#pragma unroll
                for (int r = 0; r < S::RT; ++r) {
                    const int64_t j = row0 + r;
                    if (j < row_end)
                        p.uT[i * p.d_out + j] = uacc[r];
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------
cudaError_t lnq_split_f(const float *F, int64_t d, int groups, __nv_bfloat16 *Fp, cudaStream_t s)
{
    const int64_t total = d * pieces_stride(d) * groups;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 32)
        blocks = 148 * 32;
    KernelTimer timer("lnq_split_f", s);
    split_f_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(F, d, groups, Fp);
    return cudaGetLastError();
}

// Tensor map over the pieces Fp [groups * 3][d][ld]: 64 x 128 (column x row) bf16 boxes,
// 128-byte swizzle; reads outside d x d return zeros.
bool encode_f_pieces(CUtensorMap *map, const __nv_bfloat16 *Fp, int64_t d, int groups)
{
    auto encode = tensor_map_encoder();
    if (encode == nullptr)
        return false;
    const int64_t ld = pieces_stride(d);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(d),
                          static_cast<cuuint64_t>(groups) * 3};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(d * ld) * 2};
    cuuint32_t box[3] = {vg::BK, vg::BM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(Fp), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int M>
static cudaError_t launch_vgemm_m(const CUtensorMap &map, VgParams p, int num_sms, cudaStream_t s,
                                  const char *name)
{
    using S = VgShape<M>;
    p.row_tiles_per_group = static_cast<int>((p.rows_per_group + S::RT - 1) / S::RT);
    p.i_tiles = static_cast<int>((p.d + vg::BM - 1) / vg::BM);
    const int64_t groups = p.d_out / p.rows_per_group;
    p.num_tiles = static_cast<int>(groups * p.row_tiles_per_group * p.i_tiles);
    const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    cudaError_t e = cudaFuncSetAttribute(lnq_vgemm_kernel<M>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(S::SMEM));
    if (e != cudaSuccess)
        return e;
    KernelTimer timer(name, s);
    lnq_vgemm_kernel<M><<<grid, vg::NUM_THREADS, S::SMEM, s>>>(map, p);
    return cudaGetLastError();
}

// m in {2,4,8,16}: V and uT for every row; m == 0: uT = F r only.
cudaError_t lnq_vgemm(const __nv_bfloat16 *Fp, int groups, const uint8_t *Q, const float *W,
                      const float *C, float *V, float *uT, int64_t d, int64_t d_out, int m,
                      bool residual_only, DeviceErr err, int num_sms, cudaStream_t s)
{
    CUtensorMap map;
    if (!encode_f_pieces(&map, Fp, d, groups))
        return cudaErrorInvalidValue;
    VgParams p{};
    p.Q = Q;
    p.W = W;
    p.C = C;
    p.V = V;
    p.uT = uT;
    p.d = d;
    p.d_out = d_out;
    p.rows_per_group = d_out / groups;
    p.m = m;
    p.err = err;
    if (residual_only)
        return launch_vgemm_m<0>(map, p, num_sms, s, "lnq_residual_gemm");
    switch (m) {
    case 2: return launch_vgemm_m<2>(map, p, num_sms, s, "lnq_vgemm");
    case 4: return launch_vgemm_m<4>(map, p, num_sms, s, "lnq_vgemm");
    case 8: return launch_vgemm_m<8>(map, p, num_sms, s, "lnq_vgemm");
    case 16: return launch_vgemm_m<16>(map, p, num_sms, s, "lnq_vgemm");
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
