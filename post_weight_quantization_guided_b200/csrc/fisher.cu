// fisher.cu -- guided Fisher blocks F_g = alpha * X^T diag(s_g) X on B200 (sm_100a).
//
// Source: "GuidedQuant" (jinukkim.me blog), GuidedQuant section, third equation (the
// gradient-weighted output error and its per-output-channel Fisher blocks
// F_j = (1/n) X^T diag(G_:,j^2) X) and the sentence after it (blocks are grouped and averaged
// within each group, so F_g uses s_g[t] = mean_{j in g} G[t,j]^2).
//
// Kernels:
//   token_stats_kernel      per token t: s_g[t] for every group (16-byte loads of G, fp32 sums),
//                           M_t = max_i |X[t,i]|, and per group the maximum of s_g[t] M_t^2.
//   guided_operands_kernel  A = X scaled by a power of two per token (exact in fp16) and
//                           B_g = fp16(s_g * X) scaled by powers of two (one rounding, 2^-11
//                           relative), so that F_g = alpha * Pi_g * A^T B_g. Keeping X exact on
//                           one side and fp16 on the other bounds the error of every F entry by
//                           about 5e-4 * sqrt(F_ii F_kk) even for a single token; bf16 on both
//                           sides can reach 8e-3.
//   fisher_syrk_kernel      persistent tcgen05 GEMM over the upper-triangle tiles of every F_g.
//                           TMA brings 64(t) x 64(i) boxes of A and B_g into shared memory in the
//                           128-byte-swizzled MN-major layout (no transpose of X is needed); one
//                           thread issues tcgen05.mma.kind::f16 (M=128, N=256, K=16) into a TMEM
//                           accumulator; four epilogue warps read TMEM, scale and write the tile
//                           and its mirror image. Two TMEM accumulators let the epilogue of one
//                           tile overlap the main loop of the next.
// Without gradients (G == NULL) the product is X^T X: A = B = X in bf16, no preparation pass.
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

// One warp per token t: S[g][t] = mean_{j in g} G[t,j]^2 for every group, M[t] = max_i |X[t,i]|,
// and pimax[g] = max over tokens of S[g][t] * M[t]^2 (positive floats compare as their bits).
__global__ void token_stats_kernel(const __nv_bfloat16 *__restrict__ X,
                                   const __nv_bfloat16 *__restrict__ G, int64_t n, int64_t d,
                                   int64_t d_out, int groups, float *__restrict__ S,
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
            S[static_cast<int64_t>(g) * n + t] = sg;
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

// Operands of the guided product, one thread per 8 consecutive elements of a token row:
//   A[t][:]    = fp16(X[t][:] / P_t),                          P_t = pow2_ceil(M[t])  (exact)
//   B[g][t][:] = fp16(X[t][:] * S[g][t] * P_t / Pi_g),         Pi_g = pow2_ceil(pimax[g])
// so that A[t][i] * B[g][t][k] = s_g[t] X[t][i] X[t][k] / Pi_g with one fp16 rounding, |A| <= 1
// and |B| <= 2. The GEMM epilogue multiplies by alpha * Pi_g.
__global__ void guided_operands_kernel(const __nv_bfloat16 *__restrict__ X,
                                       const float *__restrict__ S, const float *__restrict__ M,
                                       const unsigned *__restrict__ pimax, int64_t n, int64_t d,
                                       int groups, __half *__restrict__ A, __half *__restrict__ B)
{
    const int64_t vec_per_row = d / 8;
    const int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (v >= n * vec_per_row)
        return;
    const int64_t t = v / vec_per_row;
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(X) + v);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
    float2 f[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        f[e] = __bfloat1622float2(h[e]);
    const float Pt = pow2_ceil(M[t]);
    const float inv = 1.f / Pt;  // exact: Pt is a power of two
    uint4 out;
    __half2 *o = reinterpret_cast<__half2 *>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e)
        o[e] = __floats2half2_rn(f[e].x * inv, f[e].y * inv);
    reinterpret_cast<uint4 *>(A)[v] = out;
    for (int g = 0; g < groups; ++g) {
        const float factor = S[static_cast<int64_t>(g) * n + t] * Pt / pow2_ceil(__uint_as_float(pimax[g]));
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[e] = __floats2half2_rn(f[e].x * factor, f[e].y * factor);
        reinterpret_cast<uint4 *>(B + static_cast<int64_t>(g) * n * d)[v] = out;
    }
}

// ------------------------------------------------------------------------------------------
// tcgen05 SYRK over upper-triangle tiles
// ------------------------------------------------------------------------------------------
namespace syrk {
constexpr int BM = 128;          // tile rows (i), TMEM lanes
constexpr int BN = 256;          // tile columns (k), TMEM columns per accumulator
constexpr int BK = 64;           // tokens per pipeline stage
constexpr int STAGES = 4;
constexpr int BOX = 64;          // TMA box: 64 elements (128 B) along i/k  x  64 tokens
constexpr int BOX_BYTES = BOX * BK * 2;                  // 8 KB
constexpr int A_BYTES = (BM / BOX) * BOX_BYTES;          // 16 KB
constexpr int B_BYTES = (BN / BOX) * BOX_BYTES;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;           // 48 KB
constexpr int NUM_THREADS = 192;                         // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int TMEM_COLS = 2 * BN;                        // two accumulators
constexpr size_t SMEM_BYTES = static_cast<size_t>(STAGES) * STAGE_BYTES + 1024 /*align*/ + 256;
}  // namespace syrk

struct SyrkParams {
    float *F;            // [groups][d][d]
    const unsigned *pimax;  // [groups] per-group operand scale (guided), or nullptr
    int64_t n, d;
    int groups;
    float alpha;
    int nbi, nbk;        // row blocks of 128, column blocks of 256
    int tiles_per_group;
    int num_tiles;
    DeviceErr err;
};

// Tile t of one group, ordered by column block then row block; only tiles that touch the upper
// triangle (row block start <= column block end) exist.
__device__ __forceinline__ void syrk_tile_coords(const SyrkParams &p, int tile, int &g, int &bi,
                                                 int &bk)
{
    g = tile / p.tiles_per_group;
    int r = tile - g * p.tiles_per_group;
    bk = 0;
    for (;;) {
        int cnt = min(2 * bk + 2, p.nbi);
        if (r < cnt)
            break;
        r -= cnt;
        ++bk;
    }
    bi = r;
}

template <bool kF16>
__global__ void __launch_bounds__(syrk::NUM_THREADS, 1)
    fisher_syrk_kernel(const __grid_constant__ CUtensorMap amap,
                       const __grid_constant__ CUtensorMap bmap, SyrkParams p)
{
    using namespace syrk;
    constexpr uint32_t IDESC = umma_idesc_f16kind(BM, BN, /*a_mn_major=*/true,
                                                  /*b_mn_major=*/true, kF16);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                  // [STAGES]
    uint64_t *empty = bars + STAGES;        // [STAGES]
    uint64_t *tfull = bars + 2 * STAGES;    // [2]
    uint64_t *tempty = bars + 2 * STAGES + 2;  // [2]
    uint64_t *drain = bars + 2 * STAGES + 4;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4 * 32);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
    }
    if (warp == 1)
        tmem_alloc(tmem_holder, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int nk = static_cast<int>((p.n + BK - 1) / BK);
    const long long limit = p.err.limit;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int fills[STAGES];
            for (int s = 0; s < STAGES; ++s)
                fills[s] = 0;
            int stage = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                int g, bi, bk;
                syrk_tile_coords(p, tile, g, bi, bk);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[stage], (fills[stage] & 1) ^ 1, limit)) {
                        raise_error(p.err, kErrTimeout, 1);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    const int t0 = kb * BK;
                    for (int b = 0; b < BM / BOX; ++b)
                        tma_load_3d(sa + b * BOX_BYTES, &amap, &full[stage], bi * BM + b * BOX, t0, 0);
                    for (int b = 0; b < BN / BOX; ++b)
                        tma_load_3d(sb + b * BOX_BYTES, &bmap, &full[stage], bk * BN + b * BOX, t0, g);
                    ++fills[stage];
                    stage = (stage + 1 == STAGES) ? 0 : stage + 1;
                }
            }
            if (!ok) {
                // Let every load already issued land before the CTA can exit.
                for (int s = 0; s < STAGES; ++s)
                    if (fills[s] > 0)
                        mbar_wait(&full[s], (fills[s] - 1) & 1, kDrainLimit);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0, uses = 0;
            uint32_t full_phase[STAGES];
            for (int s = 0; s < STAGES; ++s)
                full_phase[s] = 0;
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const int use = it >> 1;
                if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, limit)) {
                    raise_error(p.err, kErrTimeout, 2);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[stage], full_phase[stage], limit)) {
                        raise_error(p.err, kErrTimeout, 3);
                        ok = false;
                        break;
                    }
                    full_phase[stage] ^= 1u;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // 16 tokens = two 8-row groups of the 128-byte swizzle atom.
                        const uint64_t ad = umma_desc_sw128(sa + kk * 16 * 128, BOX_BYTES, 1024);
                        const uint64_t bd = umma_desc_sw128(sb + kk * 16 * 128, BOX_BYTES, 1024);
                        umma_f16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    stage = (stage + 1 == STAGES) ? 0 : stage + 1;
                }
                if (!ok)
                    break;
                umma_commit(&tfull[acc]);
                ++uses;
            }
            // Every MMA issued by this thread has completed once `drain` flips.
            umma_commit(drain);
            mbar_wait(drain, 0, kDrainLimit);
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2-5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row_in_tile = quarter * 32 + lane;
        int it = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const int use = it >> 1;
            // One lane waits and the warp follows its verdict, so the warp-collective TMEM loads
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
                p.pimax ? p.alpha * pow2_ceil(__uint_as_float(p.pimax[g])) : p.alpha;
            const int64_t i = static_cast<int64_t>(bi) * BM + row_in_tile;
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
            mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace lnq

// ------------------------------------------------------------------------------------------
// Host launcher
// ------------------------------------------------------------------------------------------
#include <cudaTypedefs.h>

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

// F_g = scale_g * A^T B_g, both triangles written, for A [n][d] and B [groups][n][d] (row-major):
//   f16 == false: A = B = X in bf16 (groups == 1), scale = alpha;
//   f16 == true:  the guided operands above, scale_g = alpha * pow2_ceil(pimax[g]).
cudaError_t fisher_syrk(const void *A, const void *B, bool f16, const unsigned *pimax, int64_t n,
                        int64_t d, int groups, float alpha, float *F, DeviceErr err,
                        cudaStream_t s, int num_sms)
{
    using namespace syrk;
    CUtensorMap amap, bmap;
    if (tensor_map_encoder() == nullptr)
        return cudaErrorNotSupported;
    if (!encode_operand(&amap, A, n, d, 1, f16) || !encode_operand(&bmap, B, n, d, groups, f16))
        return cudaErrorInvalidValue;
    SyrkParams p;
    p.F = F;
    p.pimax = pimax;
    p.n = n;
    p.d = d;
    p.groups = groups;
    p.alpha = alpha;
    p.nbi = static_cast<int>((d + BM - 1) / BM);
    p.nbk = static_cast<int>((d + BN - 1) / BN);
    p.tiles_per_group = 0;
    for (int bk = 0; bk < p.nbk; ++bk)
        p.tiles_per_group += (2 * bk + 2 < p.nbi) ? 2 * bk + 2 : p.nbi;
    p.num_tiles = p.tiles_per_group * groups;
    p.err = err;
    const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    auto kernel = f16 ? fisher_syrk_kernel<true> : fisher_syrk_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess)
        return e;
    {
        KernelTimer timer("fisher_syrk", s);
        kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(amap, bmap, p);
    }
    return cudaGetLastError();
}

}  // namespace lnq
