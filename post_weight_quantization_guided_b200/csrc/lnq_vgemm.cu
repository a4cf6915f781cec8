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
constexpr int B_STAGES = 2;                      // stage g belongs to producer group g
constexpr int NUM_THREADS = 448;                 // w0 TMA, w1 MMA, w2-5 epilogue, w6-13 operand
constexpr int PRODUCER_THREADS = 256;           // two groups of 4 warps
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
    static constexpr int STG_BYTES = 2 * RT * 64;       // codebooks of the tile's rows, per group
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
    // per producer group: the codebooks of the tile's rows
    float(*stg_c)[16] = reinterpret_cast<float(*)[16]>(b_base + B_STAGES * S::B_BYTES + BAR_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&b_full[s], PRODUCER_THREADS / 2);  // one producer group per stage
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
        // Two groups of four warps take alternate K blocks (group g fills stage g with blocks
        // kb = g, g + 2, ...), so each group has two MMA blocks' time to build one. A thread owns
        // (row, 8-coordinate chunk) items and writes, from its own loads of Q and W, the chunk of
        // every one-hot row of that row and of its three residual-piece rows, in the 128-byte
        // swizzled K-major layout. Columns beyond S::USED are never written: the epilogue ignores
        // them. The stage wait is ANDed over the group's warps so that they leave together on a
        // timeout.
        constexpr int GT = PRODUCER_THREADS / 2;
        constexpr int ITEMS = S::RT * 8;
        constexpr int IPT = (ITEMS + GT - 1) / GT;
        const int t = threadIdx.x - 6 * 32;
        const int grp = t / GT, tg = t - grp * GT;
        const int bar_id = 1 + grp;
        float(*cs)[16] = stg_c + grp * S::RT;
        const bool vec = (p.d & 7) == 0 && (reinterpret_cast<uintptr_t>(p.Q) & 7u) == 0 &&
                         (reinterpret_cast<uintptr_t>(p.W) & 15u) == 0;
        const int stage = grp;
        int uses = 0;
        bool ok = true;
        uint2 qn[IPT];   // next block's classes (0xFF outside the problem)
        float4 wn[IPT][2];
        auto fetch = [&](int64_t row0, int64_t row_end, int64_t k0) {
#pragma unroll
            for (int s2 = 0; s2 < IPT; ++s2) {
                const int e = tg + s2 * GT;
                const int r = e >> 3, c = e & 7;
                const int64_t j = row0 + r, k = k0 + 8 * c;
                qn[s2] = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
                wn[s2][0] = wn[s2][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < ITEMS && j < row_end && k < p.d) {
                    if (vec && k + 8 <= p.d) {
                        qn[s2] = *reinterpret_cast<const uint2 *>(p.Q + j * p.d + k);
                        wn[s2][0] = *reinterpret_cast<const float4 *>(p.W + j * p.d + k);
                        wn[s2][1] = *reinterpret_cast<const float4 *>(p.W + j * p.d + k + 4);
                    } else {
                        uint32_t q2[2] = {0u, 0u};
                        float wv[8];
#pragma unroll
                        for (int e8 = 0; e8 < 8; ++e8) {
                            const bool in = k + e8 < p.d;
                            q2[e8 >> 2] |= static_cast<uint32_t>(in ? p.Q[j * p.d + k + e8] : 0xFFu)
                                           << (8 * (e8 & 3));
                            wv[e8] = in ? p.W[j * p.d + k + e8] : 0.f;
                        }
                        qn[s2] = make_uint2(q2[0], q2[1]);
                        wn[s2][0] = make_float4(wv[0], wv[1], wv[2], wv[3]);
                        wn[s2][1] = make_float4(wv[4], wv[5], wv[6], wv[7]);
                    }
                }
            }
        };
        for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
            int g, it;
            int64_t row0, row_end;
            vg_tile_coords<M>(p, tile, g, row0, row_end, it);
            if (grp >= nk)
                continue;
            // the group's copy of the tile's codebooks (the previous tile's readers are done:
            // every thread passed the group's last stage wait after its last read)
            named_bar_sync(bar_id, GT);
            for (int e = tg; e < S::RT * 16; e += GT) {
                const int r = e >> 4, b = e & 15;
                const int64_t j = row0 + r;
                cs[r][b] = (j < row_end && b < p.m) ? p.C[j * p.m + b] : 0.f;
            }
            fetch(row0, row_end, static_cast<int64_t>(grp) * BK);
            named_bar_sync(bar_id, GT);
            for (int kb = grp; kb < nk; kb += 2) {
                const int mine = mbar_wait(&b_empty[stage], (uses & 1) ^ 1, limit) ? 1 : 0;
                if (!named_bar_and(bar_id, GT, mine)) {
                    if (tg == 0)
                        raise_error(p.err, kErrTimeout, 12);
                    ok = false;
                    break;
                }
                uint2 qc[IPT];
                float4 wc[IPT][2];
#pragma unroll
                for (int s2 = 0; s2 < IPT; ++s2) {
                    qc[s2] = qn[s2];
                    wc[s2][0] = wn[s2][0];
                    wc[s2][1] = wn[s2][1];
                }
                if (kb + 2 < nk)
                    fetch(row0, row_end, static_cast<int64_t>(kb + 2) * BK);
                uint8_t *sb = b_base + stage * S::B_BYTES;
#pragma unroll
                for (int s2 = 0; s2 < IPT; ++s2) {
                    const int e = tg + s2 * GT;
                    if (e >= ITEMS)
                        continue;
                    const int r = e >> 3, c = e & 7;
                    // residual pieces of the chunk's 8 coordinates
                    const float wv[8] = {wc[s2][0].x, wc[s2][0].y, wc[s2][0].z, wc[s2][0].w,
                                         wc[s2][1].x, wc[s2][1].y, wc[s2][1].z, wc[s2][1].w};
                    uint32_t pk[3][4] = {};
#pragma unroll
                    for (int e8 = 0; e8 < 8; ++e8) {
                        const uint32_t qv = ((e8 < 4 ? qc[s2].x : qc[s2].y) >> (8 * (e8 & 3))) & 0xFFu;
                        float p0 = 0.f, p1 = 0.f, p2 = 0.f;
                        if (qv != 0xFFu)
                            split3(cs[r][qv & (p.m - 1)] - wv[e8], p0, p1, p2);
                        const int sh = 16 * (e8 & 1);
                        pk[0][e8 >> 1] |= static_cast<uint32_t>(bf16_bits(p0)) << sh;
                        pk[1][e8 >> 1] |= static_cast<uint32_t>(bf16_bits(p1)) << sh;
                        pk[2][e8 >> 1] |= static_cast<uint32_t>(bf16_bits(p2)) << sh;
                    }
#pragma unroll
                    for (int pc = 0; pc < 3; ++pc) {
                        const int n = S::ONEHOT + 3 * r + pc;
                        *reinterpret_cast<uint4 *>(sb + n * 128 + ((c ^ (n & 7)) << 4)) =
                            make_uint4(pk[pc][0], pk[pc][1], pk[pc][2], pk[pc][3]);
                    }
                    if constexpr (M > 0) {
#pragma unroll
                        for (int b = 0; b < M; ++b) {
                            const int n = r * M + b;
                            const uint32_t bbbb = 0x01010101u * static_cast<uint32_t>(b);
                            const uint32_t m0 = __vcmpeq4(qc[s2].x, bbbb), m1 = __vcmpeq4(qc[s2].y, bbbb);
                            // byte e of the mask (0xFF or 0) -> bf16 1.0 (0x3F80) or 0, half-word e
                            *reinterpret_cast<uint4 *>(sb + n * 128 + ((c ^ (n & 7)) << 4)) =
                                make_uint4(__byte_perm(m0, 0u, 0x1100) & 0x3F803F80u,
                                           __byte_perm(m0, 0u, 0x3322) & 0x3F803F80u,
                                           __byte_perm(m1, 0u, 0x1100) & 0x3F803F80u,
                                           __byte_perm(m1, 0u, 0x3322) & 0x3F803F80u);
                        }
                    }
                }
                // make the generic-proxy writes visible to the tensor core (async proxy)
                fence_proxy_async_smem();
                mbar_arrive(&b_full[stage]);
                ++uses;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // Per K block: wait for the right operand, then for each piece wait for its A slot, issue
        // four K=16 MMAs and release the slot; release the right-operand stage after the block.
        if (lane == 0) {
            int slot = 0;
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
                    const int bstage = kb & 1;  // K block kb comes from producer group kb & 1
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
