// fisher.cu -- guided Fisher blocks F_g = alpha * X^T diag(s_g) X on B200 (sm_100a).
//
// Source: "GuidedQuant" (jinukkim.me blog), GuidedQuant section, third equation (the
// gradient-weighted output error and its per-output-channel Fisher blocks
// F_j = (1/n) X^T diag(G_:,j^2) X) and the sentence after it (blocks are grouped and averaged
// within each group, so F_g uses s_g[t] = mean_{j in g} G[t,j]^2).
//
// Kernels:
//   token_stats_kernel   per token t: s_g[t] for every group (16-byte loads of G, fp32 sums),
//                        M_t = max_i |X[t,i]|, and per group the maximum of s_g[t] M_t^2.
//   token_scales_kernel  per token t: the two operand factors below, in place of s_g[t] and M_t.
//   fisher_syrk_kernel   persistent tcgen05 GEMM over the upper-triangle 256 x 256 tiles of every
//                        F_g, two CTAs (a cluster pair on two SMs) per tile. Per stage of 64
//                        tokens each CTA holds its 128 rows of the left operand and its 128 of the
//                        tile's 256 columns of the right operand, in the 128-byte-swizzled
//                        MN-major layout (64(t) x 64(i) boxes; X is never transposed). The even
//                        CTA's thread issues tcgen05.mma.cta_group::2.kind::f16 (M=256, N=256,
//                        K=16); each CTA's four epilogue warps read its 128 rows from TMEM, scale
//                        them and write them and their mirror image. Two TMEM accumulators let the
//                        epilogue of one tile overlap the main loop of the next.
//     guided (G given):  the diag(s_g) scaling is fused into the operand load. TMA brings the
//                        stage's X tiles (bf16, the same boxes as the plain path) and the stage's
//                        64 per-token factors of both operands into the stage; four groups of four
//                        converter warps, each on every fourth stage, then rewrite every
//                        16-byte chunk in place as fp16 (same swizzled
//                        position: the chunk's row is its token):
//                          A[t][i] = X[t][i] / P_t                  (P_t = pow2_ceil(M_t), exact)
//                          B[t][k] = fp16(X[t][k] * s_g[t] P_t / Pi_g)   (Pi_g = pow2_ceil(max_t
//                                                                    s_g[t] M_t^2), one rounding)
//                        so that A^T B = X^T diag(s_g) X / Pi_g with |A| <= 1, |B| <= 2, and every
//                        entry within about 5e-4 sqrt(F_ii F_kk) even for a single token (bf16 on
//                        both sides can reach 8e-3). No scaled copy of X is ever written to HBM.
//     plain (G == NULL): F = X^T X; TMA brings X in bf16 (exact products) for both operands.
#include <cuda_fp16.h>

#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

// ------------------------------------------------------------------------------------------
// Per-token statistics: s_g[t] and the row maximum M_t = max_i |X[t,i]|
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float sum_squares_bf16(const __nv_bfloat16 *__restrict__ p, int64_t len,
                                                  int lane)
{
    float acc = 0.f;
    if ((reinterpret_cast<uintptr_t>(p) & 15u) == 0 && (len & 7) == 0) {
        const uint4 *v = reinterpret_cast<const uint4 *>(p);
        for (int64_t k = lane; k < len / 8; k += 32) {
            uint4 x = __ldg(v + k);
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2 f = __bfloat1622float2(h[e]);
                acc = fmaf(f.x, f.x, acc);
                acc = fmaf(f.y, f.y, acc);
            }
        }
    } else {
        for (int64_t k = lane; k < len; k += 32) {
            float f = __bfloat162float(p[k]);
            acc = fmaf(f, f, acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// One warp per token t: S[g][t] = mean_{j in g} G[t,j]^2 for every group (row stride ld),
// M[t] = max_i |X[t,i]|, and pimax[g] = max over tokens of S[g][t] * M[t]^2 (positive floats compare
// as their bits).
__global__ void token_stats_kernel(const __nv_bfloat16 *__restrict__ X,
                                   const __nv_bfloat16 *__restrict__ G, int64_t n, int64_t ld,
                                   int64_t d, int64_t d_out, int groups, float *__restrict__ S,
                                   float *__restrict__ M, unsigned *__restrict__ pimax)
{
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= n)
        return;
    const uint4 *xv = reinterpret_cast<const uint4 *>(X + t * d);
    float mx = 0.f;
    for (int64_t k = lane; k < d / 8; k += 32) {
        uint4 x = __ldg(xv + k);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(h[e]);
            mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0)
        M[t] = mx;
    const int64_t R = d_out / groups;
    for (int g = 0; g < groups; ++g) {
        const float sg = sum_squares_bf16(G + t * d_out + g * R, R, lane) / static_cast<float>(R);
        if (lane == 0) {
            S[static_cast<int64_t>(g) * ld + t] = sg;
            atomicMax(&pimax[g], __float_as_uint(sg * mx * mx));
        }
    }
}

// Smallest power of two >= v for finite v > 0; 1 for v == 0.
__device__ __forceinline__ float pow2_ceil(float v)
{
    if (!(v > 0.f))
        return 1.f;
    const unsigned u = __float_as_uint(v);
    if ((u & 0x007FFFFFu) == 0u)
        return v;
    return __uint_as_float((u & 0x7F800000u) + 0x00800000u);
}

// Per-token operand factors of the guided product, in place of the statistics they come from:
//   M[t]    <- 1 / P_t,                    P_t = pow2_ceil(M_t)           (exact)
//   S[g][t] <- S[g][t] * P_t / Pi_g,       Pi_g = pow2_ceil(pimax[g])
// so that the left operand X[t][:] / P_t is exact in fp16 (|.| <= 1), the right operand
// fp16(X[t][:] * S[g][t] P_t / Pi_g) is rounded once (|.| <= 2), and their product is
// s_g[t] X[t][i] X[t][k] / Pi_g. One thread per token of the padded range: tokens n .. ld - 1
// get zero factors (the SYRK's stages copy whole blocks of 64).
__global__ void token_scales_kernel(int64_t n, int64_t ld, int groups, float *__restrict__ S,
                                    float *__restrict__ M, const unsigned *__restrict__ pimax)
{
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= ld)
        return;
    if (t >= n) {
        for (int g = 0; g < groups; ++g)
            S[static_cast<int64_t>(g) * ld + t] = 0.f;
        M[t] = 0.f;
        return;
    }
    const float Pt = pow2_ceil(M[t]);
    for (int g = 0; g < groups; ++g)
        S[static_cast<int64_t>(g) * ld + t] =
            S[static_cast<int64_t>(g) * ld + t] * Pt / pow2_ceil(__uint_as_float(pimax[g]));
    M[t] = 1.f / Pt;
}

// ------------------------------------------------------------------------------------------
// tcgen05 SYRK over upper-triangle tiles, two CTAs (a cluster pair on two SMs) per tile
// ------------------------------------------------------------------------------------------
namespace syrk {
constexpr int BM = 128;          // tile rows (i) per CTA: TMEM lanes; the pair covers 2 BM
constexpr int PM = 2 * BM;       // rows of a pair tile
constexpr int BN = 256;          // tile columns (k), TMEM columns per accumulator
constexpr int HALF = BN / 2;     // columns of the right operand each CTA holds
constexpr int BK = 64;           // tokens per pipeline stage
constexpr int STAGES = 6;
constexpr int BOX = 64;          // operand box: 64 elements (128 B) along i/k  x  BK tokens
constexpr int BOX_BYTES = BOX * BK * 2;                  // 8 KB
constexpr int A_BYTES = (BM / BOX) * BOX_BYTES;          // 16 KB
constexpr int B_BYTES = (HALF / BOX) * BOX_BYTES;        // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;           // 32 KB per CTA
// warp 0 TMA, warp 1 MMA, warps 2-5 epilogue, then (guided) CONV_GROUPS groups of four converter
// warps; group k converts the stages of fills k, k + CONV_GROUPS, ...
constexpr int CONV_GROUPS = 4;
constexpr int GROUP_THREADS = 128;
constexpr int CONV_THREADS = CONV_GROUPS * GROUP_THREADS;
constexpr int GROUP_WARPS = GROUP_THREADS / 32;
constexpr int SCALE_BYTES = 2 * BK * 4;                  // the stage's factors of both operands
__host__ __device__ constexpr int num_threads(bool guided) { return guided ? 192 + CONV_THREADS : 192; }
constexpr int TMEM_COLS = 2 * BN;                        // two accumulators
constexpr int NUM_BARS = 3 * STAGES + 5;                 // full, empty, raw_full; tfull, tempty, drain
constexpr int BAR_BYTES = (NUM_BARS * 8 + 4 + 15) / 16 * 16;   // + the TMEM address holder
constexpr size_t SMEM_BYTES = static_cast<size_t>(STAGES) * (STAGE_BYTES + SCALE_BYTES) +
                              1024 /*align*/ + BAR_BYTES;
constexpr uint16_t PAIR = 0x3;                           // both CTAs of the cluster
constexpr long long kPairDrainLimit = 1LL << 22;
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert((A_BYTES / 16) % GROUP_THREADS == 0 && A_BYTES == B_BYTES, "converter tiling");
}  // namespace syrk

struct SyrkParams {
    float *F;            // [groups][d][d]
    const float *bfac;   // [groups][ld] right-operand factor s_g[t] P_t / Pi_g (guided)
    const float *ainv;   // [ld] left-operand factor 1 / P_t (guided)
    int64_t ld;          // n rounded up to a multiple of 64 (guided factor rows)
    const unsigned *pimax;  // [groups] per-group operand scale (guided), or nullptr
    int64_t n, d;
    int groups;
    float alpha;
    int nb;              // blocks of 256 along i and k
    int tiles_per_group; // nb (nb + 1) / 2: the blocks (bi, bk) with bi <= bk
    int num_tiles;
    DeviceErr err;
};

// Pair tile t of one group, ordered by column block then row block: (bi, bk) with bi <= bk.
__device__ __forceinline__ void syrk_tile_coords(const SyrkParams &p, int tile, int &g, int &bi,
                                                 int &bk)
{
    g = tile / p.tiles_per_group;
    int r = tile - g * p.tiles_per_group;
    bk = 0;
    while (r > bk) {
        r -= bk + 1;
        ++bk;
    }
    bi = r;
}

// 8 bf16 values times `scale`, rounded once to fp16: each pair is widened to fp32 (exact), both
// halves are multiplied by one packed fp32 multiply (round to nearest, as two scalar ones) and
// rounded to fp16 by one packed conversion.
__device__ __forceinline__ uint4 scale_bf16x8_to_f16(uint4 x, float scale)
{
    const uint64_t sc2 = (static_cast<uint64_t>(__float_as_uint(scale)) << 32) | __float_as_uint(scale);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        // low element in the low word, high element in the high word
        const uint64_t pair = (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32) | (w[e] << 16);
        uint64_t prod;
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(prod) : "l"(pair), "l"(sc2));
        asm("cvt.rn.f16x2.f32 %0, %1, %2;"
            : "=r"(r[e])
            : "f"(__uint_as_float(static_cast<uint32_t>(prod >> 32))),
              "f"(__uint_as_float(static_cast<uint32_t>(prod))));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

template <bool kGuided>
__device__ __forceinline__ void fisher_syrk_body(const CUtensorMap &amap, const CUtensorMap &bmap,
                                                 const SyrkParams &p)
{
    using namespace syrk;
    constexpr uint32_t IDESC = umma_idesc_f16kind(PM, BN, /*a_mn_major=*/true,
                                                  /*b_mn_major=*/true, kGuided);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    float *scales = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES);  // [STAGES][2][BK]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * (STAGE_BYTES + SCALE_BYTES));
    uint64_t *full = bars;                  // [STAGES] (the even CTA's counts both CTAs' fills)
    uint64_t *empty = bars + STAGES;        // [STAGES]
    uint64_t *tfull = bars + 2 * STAGES;    // [2]
    uint64_t *tempty = bars + 2 * STAGES + 2;  // [2] (the even CTA's counts both epilogues)
    uint64_t *drain = bars + 2 * STAGES + 4;
    uint64_t *raw_full = bars + 2 * STAGES + 5;  // [STAGES] guided: this CTA's copies landed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 3 * STAGES + 5);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cr = cluster_ctarank();  // 0: issues the pair's MMAs; 1: its peer
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // guided: one arrival per converter warp of both CTAs; plain: the even CTA's
            // expect_tx arrival, with the TMA bytes of both CTAs
            mbar_init(&full[s], kGuided ? 2 * GROUP_WARPS : 1);
            mbar_init(&empty[s], 1);
            mbar_init(&raw_full[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * 4 * 32);   // the epilogues of both CTAs
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
    }
    if (warp == 1)
        tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int nk = static_cast<int>((p.n + BK - 1) / BK);
    const long long limit = p.err.limit;

    if (warp == 0 && kGuided) {
        // ---------------------------------------------------------------- TMA producer (guided)
        // Per stage: this CTA's X tiles of both operands (bf16) and the stage's factors, counted
        // on this CTA's raw_full barrier; the converters turn them into the operands in place.
        if (lane == 0) {
            int stage = 0, use = 0;
            uint32_t used = 0u;
            bool ok = true;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, bi, bk;
                syrk_tile_coords(p, tile, g, bi, bk);
                const int i0 = bi * PM + static_cast<int>(cr) * BM;
                const int k0 = bk * BN + static_cast<int>(cr) * HALF;
                const float *bf = p.bfac + static_cast<int64_t>(g) * p.ld;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], (use & 1) ^ 1, limit)) {
                        raise_error(p.err, kErrTimeout, 1);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    float *sc = scales + stage * 2 * BK;
                    mbar_arrive_expect_tx(&raw_full[stage], STAGE_BYTES + SCALE_BYTES);
                    const int t0 = kb * BK;
                    for (int b = 0; b < BM / BOX; ++b)
                        tma_load_3d(sa + b * BOX_BYTES, &amap, &raw_full[stage], i0 + b * BOX, t0, 0);
                    for (int b = 0; b < HALF / BOX; ++b)
                        tma_load_3d(sa + A_BYTES + b * BOX_BYTES, &amap, &raw_full[stage],
                                    k0 + b * BOX, t0, 0);
                    bulk_load(sc, p.ainv + t0, BK * 4, &raw_full[stage]);
                    bulk_load(sc + BK, bf + t0, BK * 4, &raw_full[stage]);
                    used |= 1u << stage;
                    if (++stage == STAGES) {
                        stage = 0;
                        ++use;
                    }
                }
            }
            if (!ok) {
                // let this CTA's copies land before it exits: wait for the last armed phase of
                // every stage (its parity is that of the number of completed uses)
                for (int s = 0; s < STAGES; ++s) {
                    if (!((used >> s) & 1u))
                        continue;
                    const int last_use = s < stage ? use : use - 1;
                    mbar_wait(&raw_full[s], last_use & 1, kDrainLimit);
                }
            }
        }
    } else if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (plain)
        // Per stage: this CTA's 128 rows of A and its 128 of the tile's 256 columns of B, the
        // bytes of both CTAs counted on the even CTA's barrier (armed there for both).
        if (lane == 0) {
            uint32_t fpar = 0u, fused = 0u;  // per stage: parity of the fills, ever filled
            int stage = 0;
            bool ok = true;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int g, bi, bk;
                syrk_tile_coords(p, tile, g, bi, bk);
                const int i0 = bi * PM + static_cast<int>(cr) * BM;
                const int k0 = bk * BN + static_cast<int>(cr) * HALF;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], ((fpar >> stage) & 1u) ^ 1u, limit)) {
                        raise_error(p.err, kErrTimeout, 1);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    if (cr == 0)
                        mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
                    const uint32_t fb = cluster_addr(&full[stage], 0);
                    const int t0 = kb * BK;
                    for (int b = 0; b < BM / BOX; ++b)
                        tma_load_3d_pair(sa + b * BOX_BYTES, &amap, fb, i0 + b * BOX, t0, 0);
                    for (int b = 0; b < HALF / BOX; ++b)
                        tma_load_3d_pair(sb + b * BOX_BYTES, &bmap, fb, k0 + b * BOX, t0, g);
                    fpar ^= 1u << stage;
                    fused |= 1u << stage;
                    stage = (stage + 1 == STAGES) ? 0 : stage + 1;
                }
            }
            if (!ok) {
                // let this CTA's copies land before the pair exits: the even CTA waits for the
                // last phase of each stage it armed; the odd CTA's copies are counted there, so it
                // waits a fixed time
                if (cr == 0) {
                    for (int s = 0; s < STAGES; ++s)
                        if ((fused >> s) & 1u)
                            mbar_wait(&full[s], ((fpar >> s) & 1u) ^ 1u, kPairDrainLimit);
                } else {
                    const long long c0 = clock64();
                    while (clock64() - c0 < kPairDrainLimit) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (even CTA)
        if (cr == 0 && lane == 0) {
            int stage = 0;
            uint32_t fph = 0u;  // per stage: phase parity
            bool ok = true;
            int it = 0;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs, ++it) {
                const int acc = it & 1;
                const int use = it >> 1;
                if (!mbar_wait_cluster(&tempty[acc], (use & 1) ^ 1, limit)) {
                    raise_error(p.err, kErrTimeout, 2);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    const bool got = kGuided ? mbar_wait_cluster(&full[stage], (fph >> stage) & 1u, limit)
                                             : mbar_wait(&full[stage], (fph >> stage) & 1u, limit);
                    if (!got) {
                        raise_error(p.err, kErrTimeout, 3);
                        ok = false;
                        break;
                    }
                    fph ^= 1u << stage;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // 16 tokens = two 8-row groups of the 128-byte swizzle atom.
                        const uint64_t ad = umma_desc_sw128(sa + kk * 16 * 128, BOX_BYTES, 1024);
                        const uint64_t bd = umma_desc_sw128(sb + kk * 16 * 128, BOX_BYTES, 1024);
                        umma_f16_pair(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit_pair(&empty[stage], PAIR);
                    stage = (stage + 1 == STAGES) ? 0 : stage + 1;
                }
                if (!ok)
                    break;
                umma_commit_pair(&tfull[acc], PAIR);
            }
            // Every MMA issued by this thread has completed once `drain` flips.
            umma_commit_pair(drain, 0x1);
            mbar_wait(drain, 0, kDrainLimit);
        }
    } else if (warp < 6) {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row_in_tile = static_cast<int>(cr) * BM + quarter * 32 + lane;
        const uint32_t tempty_leader[2] = {cluster_addr(&tempty[0], 0), cluster_addr(&tempty[1], 0)};
        int it = 0;
        for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
            const int acc = it & 1;
            const int use = it >> 1;
            // One lane waits and the warp follows its outcome, so the warp-collective TMEM loads
            // below are executed by all 32 lanes or by none.
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait(&tfull[acc], use & 1, limit) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0)
                    raise_error(p.err, kErrTimeout, 4);
                break;
            }
            __syncwarp();
            tc_fence_after();
            int g, bi, bk;
            syrk_tile_coords(p, tile, g, bi, bk);
            float *Fg = p.F + static_cast<int64_t>(g) * p.d * p.d;
            const float scale =
                kGuided ? p.alpha * pow2_ceil(__uint_as_float(p.pimax[g])) : p.alpha;
            const int64_t i = static_cast<int64_t>(bi) * PM + row_in_tile;
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                float v[32];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(acc * BN + chunk * 32);
                tmem_ld_32x32b_x32(taddr, v);
                const int64_t k0 = static_cast<int64_t>(bk) * BN + chunk * 32;
                if (i < p.d) {
                    // the tile itself: element (i, k) for k >= i
                    float *rowp = Fg + i * p.d;
                    if (k0 >= i && k0 + 32 <= p.d) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(rowp + k0 + e) =
                                make_float4(scale * v[e], scale * v[e + 1],
                                            scale * v[e + 2], scale * v[e + 3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int64_t k = k0 + e;
                            if (k >= i && k < p.d)
                                rowp[k] = scale * v[e];
                        }
                    }
                    // the mirror: element (k, i) for k > i; lanes are consecutive i (coalesced)
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int64_t k = k0 + e;
                        if (k > i && k < p.d)
                            Fg[k * p.d + i] = scale * v[e];
                    }
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader[acc]);
        }
    } else if constexpr (kGuided) {
        // ---------------------------------------------------------------- operand converters
        // Group k converts the stages of fills k, k + CONV_GROUPS, ... once this CTA's copies have
        // landed: every 16-byte chunk of the two operand halves (8 coordinates of one token row of
        // a box) is rewritten in place as fp16, scaled by its token's factor; the chunk's token is
        // its row in the box, whatever the swizzle. Thread q of a group takes chunks q, q + 128, ...
        // of each operand. Each warp arrives once on the even CTA's barrier.
        const int cq = threadIdx.x - 6 * 32;
        const int grp = cq / GROUP_THREADS;
        const int q = cq % GROUP_THREADS;
        constexpr int PER_THREAD = A_BYTES / 16 / GROUP_THREADS;  // chunks per operand
        const uint32_t full_leader_base = cluster_addr(&full[0], 0);
        const int total = ((p.num_tiles - pair + npairs - 1) / npairs) * nk;  // this pair's stages
        for (int f = grp; f < total; f += CONV_GROUPS) {
            const int stage = f % STAGES, use = f / STAGES;
            int got = 0;
            if (lane == 0)
                got = mbar_wait(&raw_full[stage], use & 1, limit) ? 1 : 0;
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got) {
                if (lane == 0)
                    raise_error(p.err, kErrTimeout, 5);
                break;
            }
            uint8_t *sa = smem + stage * STAGE_BYTES;
            const float *sc = scales + stage * 2 * BK;
#pragma unroll
            for (int opnd = 0; opnd < 2; ++opnd) {
                uint8_t *base = sa + opnd * A_BYTES;
                uint4 x[PER_THREAD];
#pragma unroll
                for (int k = 0; k < PER_THREAD; ++k)
                    x[k] = *reinterpret_cast<const uint4 *>(base + (q + GROUP_THREADS * k) * 16);
#pragma unroll
                for (int k = 0; k < PER_THREAD; ++k) {
                    const int c = q + GROUP_THREADS * k;     // chunk of this operand's half stage
                    const int tok = (c >> 3) & (BK - 1);      // its row in its BK-row box
                    *reinterpret_cast<uint4 *>(base + c * 16) =
                        scale_bf16x8_to_f16(x[k], sc[opnd * BK + tok]);
                }
            }
            fence_proxy_async_smem();  // the stores become visible to the tensor core
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(full_leader_base + static_cast<uint32_t>(stage * 8));
        }
    }

    // Both CTAs stay until the pair is done: the MMAs read both CTAs' shared memory and the
    // copies, producers and epilogues of both signal barriers in the even CTA.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// The two instantiations: plain (192 threads) and guided (704 threads: 22 warps, at most six on
// each of the SM's four register-file quarters, so at most 80 registers per thread).
__global__ void __launch_bounds__(syrk::num_threads(false), 1)
    fisher_syrk_plain_kernel(const __grid_constant__ CUtensorMap amap,
                             const __grid_constant__ CUtensorMap bmap, SyrkParams p)
{
    fisher_syrk_body<false>(amap, bmap, p);
}

__global__ void __launch_bounds__(syrk::num_threads(true), 1)
    fisher_syrk_guided_kernel(const __grid_constant__ CUtensorMap amap,
                              const __grid_constant__ CUtensorMap bmap, SyrkParams p)
{
    fisher_syrk_body<true>(amap, bmap, p);
}

}  // namespace lnq

// ------------------------------------------------------------------------------------------
// Host launcher
// ------------------------------------------------------------------------------------------
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

namespace lnq {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

static bool encode_operand(CUtensorMap *map, const void *base, int64_t n, int64_t d, int groups,
                           bool f16)
{
    using namespace syrk;
    auto encode = tensor_map_encoder();
    if (encode == nullptr)
        return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                          static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n * d) * 2};
    cuuint32_t box[3] = {BOX, BK, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// F_g = scale_g * (operands)^T (operands), both triangles written:
//   S == nullptr: F = alpha X^T X, X read by TMA in bf16 (groups == 1);
//   otherwise:    the guided blocks, operands converted in the stages from X and the factors that
//                 token_scales_kernel left in S (right, row stride ld) and M (left), ld >= n a
//                 multiple of BK, scale_g = alpha * pow2_ceil(pimax[g]).
cudaError_t fisher_syrk(const __nv_bfloat16 *X, const float *S, const float *M,
                        const unsigned *pimax, int64_t n, int64_t ld, int64_t d, int groups,
                        float alpha, float *F, DeviceErr err, cudaStream_t s, int num_sms)
{
    using namespace syrk;
    const bool guided = S != nullptr;
    CUtensorMap amap, bmap;
    if (tensor_map_encoder() == nullptr)
        return cudaErrorNotSupported;
    if (!encode_operand(&amap, X, n, d, 1, false) || !encode_operand(&bmap, X, n, d, 1, false))
        return cudaErrorInvalidValue;
    SyrkParams p;
    p.F = F;
    p.bfac = S;
    p.ainv = M;
    p.ld = ld;
    if (guided && ld % BK != 0)
        return cudaErrorInvalidValue;   // the stages copy whole blocks of BK factors
    p.pimax = pimax;
    p.n = n;
    p.d = d;
    p.groups = groups;
    p.alpha = alpha;
    p.nb = static_cast<int>((d + PM - 1) / PM);
    p.tiles_per_group = p.nb * (p.nb + 1) / 2;
    p.num_tiles = p.tiles_per_group * groups;
    p.err = err;
    auto kernel = guided ? fisher_syrk_guided_kernel : fisher_syrk_plain_kernel;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(num_threads(guided));
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many pairs as can be resident at once (one CTA per SM)
    static int resident[2] = {0, 0};
    int &res = resident[guided ? 1 : 0];
    if (res == 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters < 1) {
            (void)cudaGetLastError();   // a failed query is not an error of this call
            clusters = num_sms / 2;
        }
        res = clusters;
    }
    int pairs = res < p.num_tiles ? res : p.num_tiles;
    if (pairs < 1)
        pairs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    {
        KernelTimer timer("fisher_syrk", s);
        e = cudaLaunchKernelEx(&cfg, kernel, amap, bmap, p);
    }
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace lnq
