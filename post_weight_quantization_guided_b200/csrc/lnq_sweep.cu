// lnq_sweep.cu -- the assignment sweep of an LNQ iteration (coordinate descent) on sm_100a.
//
// Source: "GuidedQuant" (jinukkim.me blog), LNQ section: after the codebook update, coordinate
// i = 1..d_in in turn takes the codeword minimising (w^ - w)^T F (w^ - w). With u = F r
// (r = w^ - w), moving coordinate i by delta changes the objective by delta (2 u_i + delta F_ii)
// and changes u by delta F[:, i].
//
// One CTA per 32 rows of one Fisher group. Coordinates are taken in windows of 128 (the height
// of a tensor-core tile), each window in four blocks of 32.
//   * Before a window starts, its u is assembled left-looking: the value at the start of the
//     sweep, u0 = F (c[q] - w) for the new codebook c (the residual product of lnq_vgemm.cu),
//     plus F[window][earlier coordinates] x Delta[earlier coordinates], Delta being the moves
//     made so far in this sweep. That product runs on tcgen05
//     tensor cores: F as its two fp16 pieces with a power-of-two scale per row (the operand of
//     lnq_vgemm, 22 bits per entry), Delta as two fp16 pieces with a power-of-two scale per
//     row of W (22 bits), three piece products (F2 x D2, below 2^-22 of each term, is left out)
//     accumulated in fp32 in TMEM; the scales are
//     undone exactly when the window is assembled.
//   * Delta of finished windows is kept per CTA in a global history (fp16 pieces), already in
//     the swizzled K-major layout the MMA reads, written and read back with byte-exact copies.
//   * The product for window T+1 over windows < T runs while window T is being decided; only the
//     contribution of window T itself waits for its last decision.
//   * Inside a window one warp (lane = row) decides a block of 32 coordinates: the best codeword
//     for a coordinate is the one nearest to t = w^_i - u_i / F_ii, found among the midpoints of
//     the row's sorted codebook, and the coordinate moves only if its exact change is strictly
//     negative; the block's later coordinates are corrected in registers from the 32 x 32 diagonal
//     tile of F. The four sweep warps then add the block's moves to the next block's coordinates,
//     and while warp 6 decides that block, warps 7-9 write the finished block's codes and moves,
//     correct the window's later blocks in shared memory from a 32 x 128 strip of F (one TMA box
//     per block) and start the copies for the block after.
// Warp roles: 0 TMA and bulk copies, 1 MMA issue, 2-5 window assembly (TMEM -> shared memory),
// 6-9 the sweep. Every wait is bounded; a wait that gives up sets the
// workspace error flag and its role stops, and every role drains what it has in flight.
#include <cstring>

#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

namespace sw {
constexpr int RB = 32;                    // rows per CTA (MMA N)
constexpr int WIN = 128;                  // coordinates per window (MMA M)
constexpr int BLK = 32;                   // coordinates per decision block
constexpr int NBLK = WIN / BLK;
constexpr int CH = 64;                    // coordinates per K chunk: one 128-byte bf16 swizzle row
constexpr int FPIECES = 2;                // fp16 pieces of F
constexpr int A_TILE = WIN * CH * 2;      // one fp16 piece of F[window][chunk]: 16 KB
constexpr int H_PIECE = RB * CH * 2;      // one fp16 piece of Delta[chunk][rows]: 4 KB
constexpr int DPIECES = 2;                // fp16 pieces of Delta
constexpr int H_CHUNK = DPIECES * H_PIECE;  // 8 KB
constexpr int NA = 6;                     // F piece slots
constexpr int NH = 3;                     // history chunk slots
constexpr int UW_LD = WIN + 1;            // row stride (floats) of a window's u in shared memory
constexpr int NUM_THREADS = 320;
constexpr int SWEEP_THREADS = 128;
constexpr int TMEM_COLS = 64;             // two fp32 accumulators of RB columns
constexpr int MAX_WIN = 16384 / WIN;      // d_in <= 16384
constexpr int SWEEP_BAR = 2;              // named barrier of the sweep warps
constexpr int HELP_BAR = 3;               // named barrier of sweep warps 7-9
constexpr int LEAD = 32;                  // sweep thread that issues the F strip copies

// shared memory carve-up (bytes from a 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_H = OFF_A + NA * A_TILE;
constexpr int OFF_BS = OFF_H + NH * H_CHUNK;
constexpr int OFF_STRIP = OFF_BS + 2 * H_CHUNK;
constexpr int OFF_UW = OFF_STRIP + 2 * BLK * WIN * 4;
constexpr int OFF_DL = OFF_UW + 2 * RB * UW_LD * 4;
constexpr int OFF_C = OFF_DL + 2 * BLK * RB * 4;      // moves: two blocks in flight
constexpr int OFF_QB = OFF_C + RB * 17 * 4;
constexpr int OFF_WM = OFF_QB + 2 * RB * (BLK + 8);   // codes: two blocks in flight
constexpr int OFF_TS = (OFF_WM + MAX_WIN + 15) / 16 * 16;  // [2][RB] Delta scales 2^t, 2^-t
constexpr int OFF_SRT = OFF_TS + 2 * RB * 4;               // [RB][17] sorted codebook
constexpr int OFF_ORD = OFF_SRT + RB * 17 * 4;             // [RB][16] its codeword indices
constexpr int OFF_FINV = OFF_ORD + RB * 16;                // [BLK] 1 / F_ii of the block
constexpr int OFF_FDG = OFF_FINV + BLK * 4;                // [BLK] F_ii of the block
constexpr int OFF_RM = OFF_FDG + BLK * 4;                  // [2][RB] moved-coordinate mask per row
constexpr int OFF_BAR = OFF_RM + 2 * RB * 4;
constexpr int NBARS = 2 * NA + 2 * NH + 2 + 2 + 2 + 2 + 3 + 2;
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
constexpr size_t SMEM = 1024 + OFF_MISC + 32;
static_assert(SMEM <= 232448, "shared memory");
static_assert(OFF_H % 1024 == 0 && OFF_BS % 1024 == 0, "swizzle atoms are 1024-byte aligned");
static_assert(OFF_QB % 8 == 0 && OFF_STRIP % 16 == 0, "vector accesses to the code and strip tiles");
}  // namespace sw

struct SwParams {
    const float *F;      // [groups][d][d]
    const float *U;      // [d_out][d] u = F r at the start of the sweep (codebook C, codes Q)
    const float *C;      // [d_out][m]
    uint8_t *Q;          // [d_out][d]
    uint8_t *hist;       // [CTAs][2 * windows][2][4 KB]
    const int32_t *fexp; // [groups][d] row scales of the fp16 pieces of F
    int64_t d, d_out, rows_per_group;
    int strip_tma;       // F strips by TMA (d % 4 == 0, F 16-byte aligned) or by plain loads
    int blocks_per_group, nwin;
    // work counters in the workspace header: [0] coordinates moved, [1] the sum over those moves
    // of (d - i), the entries of u that each move updates
    unsigned long long *counters;
    DeviceErr err;
};

// Sum of the positions of the set bits of a 32-bit mask.
__device__ __forceinline__ unsigned bit_position_sum(unsigned m)
{
    return __popc(m & 0xAAAAAAAAu) + 2u * __popc(m & 0xCCCCCCCCu) + 4u * __popc(m & 0xF0F0F0F0u) +
           8u * __popc(m & 0xFF00FF00u) + 16u * __popc(m & 0xFFFF0000u);
}

// The decisions of one block for one row (lane = row). With F_ii > 0, candidate a changes the
// objective by F_ii ((c_a - t)^2 - (cur - t)^2), t = cur - u_i / F_ii, so the best candidate is
// the codeword nearest to t: a binary search of the sorted codebook's midpoints, held in
// registers, halving the candidate values and midpoints at each level (selects only, no loads on
// the chain). Its change delta (2 u_i + delta F_ii) is then evaluated and the coordinate moves only
// if that is strictly negative. (F_ii = 0 gives t = -+inf, the extreme codeword, which is the best
// one for a linear change.) The later coordinates of the block are corrected in registers from
// the block's rows of the F strip. The shared-memory views are restrict-qualified, so that the
// loads of later coordinates may be issued ahead of the stores of earlier ones.
template <int M>
__device__ __forceinline__ unsigned sweep_decide_block(
    float (&ub)[sw::BLK], uint32_t (&qw)[sw::BLK / 4], const uint32_t (&qo)[sw::BLK / 4],
    const float *__restrict__ crow, const uint8_t *__restrict__ ordrow,
    const float *__restrict__ finv, const float *__restrict__ fdg, const float *__restrict__ st,
    float *__restrict__ dlcol, const float (&mid)[M > 1 ? M - 1 : 1], const float (&sv)[M],
    bool vr, int nb)
{
    using namespace sw;
    unsigned rowmask = 0u;
#pragma unroll
    for (int ii = 0; ii < BLK; ++ii) {
        const float u = ub[ii];
        const float cur = crow[(qo[ii >> 2] >> (8 * (ii & 3))) & 0xFFu];
        const float tt = fmaf(-u, finv[ii], cur);
        float V[M], Mi[M];
#pragma unroll
        for (int k = 0; k < M; ++k) {
            V[k] = sv[k];
            Mi[k] = k + 1 < M ? mid[k + 1 < M ? k : 0] : 0.f;
        }
        int pos = 0;
#pragma unroll
        for (int S = M; S > 1; S >>= 1) {
            const int h = S / 2;
            const bool up = tt > Mi[h - 1];
#pragma unroll
            for (int k = 0; k < h; ++k)
                V[k] = up ? V[k + h] : V[k];
#pragma unroll
            for (int k = 0; k + 1 < h; ++k)
                Mi[k] = up ? Mi[k + h] : Mi[k];
            pos += up ? h : 0;
        }
        const float da = V[0] - cur;
        const float D = da * fmaf(da, fdg[ii], 2.f * u);
        // a strictly negative change implies c != cur
        const bool mv = vr && ii < nb && D < 0.f;
        const float dlt = mv ? da : 0.f;
        rowmask |= (mv ? 1u : 0u) << ii;
        const int sh = 8 * (ii & 3);
        const uint32_t nq =
            (qw[ii >> 2] & ~(0xFFu << sh)) | (static_cast<uint32_t>(ordrow[pos]) << sh);
        qw[ii >> 2] = mv ? nq : qw[ii >> 2];
#pragma unroll
        for (int v = (ii + 1) / 4; v < BLK / 4; ++v) {
            const float4 f4 = *reinterpret_cast<const float4 *>(st + ii * WIN + 4 * v);
            if (4 * v > ii) ub[4 * v] = fmaf(dlt, f4.x, ub[4 * v]);
            if (4 * v + 1 > ii) ub[4 * v + 1] = fmaf(dlt, f4.y, ub[4 * v + 1]);
            if (4 * v + 2 > ii) ub[4 * v + 2] = fmaf(dlt, f4.z, ub[4 * v + 2]);
            if (4 * v + 3 > ii) ub[4 * v + 3] = fmaf(dlt, f4.w, ub[4 * v + 3]);
        }
        dlcol[ii * RB] = dlt;
    }
    return rowmask;
}

template <int M>
__global__ void __launch_bounds__(sw::NUM_THREADS, 1)
    sweep_kernel(const __grid_constant__ CUtensorMap fmap, const __grid_constant__ CUtensorMap smap,
                 SwParams p)
{
    using namespace sw;
    constexpr uint32_t IDESC = umma_idesc_f16kind(WIN, RB, false, false, /*f16=*/true);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    uint8_t *a_base = smem + OFF_A;                                  // [NA][16 KB]
    uint8_t *h_base = smem + OFF_H;                                  // [NH][12 KB]
    uint8_t *bs_base = smem + OFF_BS;                                // [2 chunks][2][4 KB]
    float *strip = reinterpret_cast<float *>(smem + OFF_STRIP);      // [2][BLK][WIN]
    float *uwb = reinterpret_cast<float *>(smem + OFF_UW);           // [2][RB][UW_LD]
    float(*dl2)[BLK][RB] = reinterpret_cast<float(*)[BLK][RB]>(smem + OFF_DL);  // [2][BLK][RB] moves
    float(*c_s)[17] = reinterpret_cast<float(*)[17]>(smem + OFF_C);         // [RB][m]
    // [2][RB][BLK + 8] codes of the current and the next block, rows 8-byte aligned
    uint8_t(*qb2)[RB][BLK + 8] = reinterpret_cast<uint8_t(*)[RB][BLK + 8]>(smem + OFF_QB);
    volatile uint8_t *wmask = smem + OFF_WM;                         // [window]: some row moved
    float *dsc = reinterpret_cast<float *>(smem + OFF_TS);            // [RB] 2^t_r of Delta row r
    float *dinv = dsc + RB;                                           // [RB] 2^-t_r
    float(*srt_s)[17] = reinterpret_cast<float(*)[17]>(smem + OFF_SRT);
    uint8_t(*ord_s)[16] = reinterpret_cast<uint8_t(*)[16]>(smem + OFF_ORD);
    float *finv_s = reinterpret_cast<float *>(smem + OFF_FINV);
    float *fdg_s = reinterpret_cast<float *>(smem + OFF_FDG);
    unsigned(*rm2)[RB] = reinterpret_cast<unsigned(*)[RB]>(smem + OFF_RM);  // [2][RB]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *a_full = bars;
    uint64_t *a_empty = a_full + NA;
    uint64_t *h_full = a_empty + NA;
    uint64_t *h_empty = h_full + NH;
    uint64_t *acc_full = h_empty + NH;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *uw_ready = acc_empty + 2;
    uint64_t *uw_free = uw_ready + 2;
    uint64_t *bs_ready = uw_free + 2;
    uint64_t *bs_free = bs_ready + 1;
    uint64_t *drain = bs_free + 1;
    uint64_t *strip_full = drain + 1;                                // [2] F strip buffers
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    // [2] per block: the OR of its rows' move masks
    volatile unsigned *mv2 = reinterpret_cast<volatile unsigned *>(smem + OFF_MISC + 16);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x / p.blocks_per_group;
    const int rb = blockIdx.x - g * p.blocks_per_group;
    const int64_t gstart = static_cast<int64_t>(g) * p.rows_per_group;
    const int64_t row0 = gstart + static_cast<int64_t>(rb) * RB;
    const int64_t row_end = min(row0 + RB, gstart + p.rows_per_group);
    const int nrows = static_cast<int>(row_end - row0);
    const int64_t d = p.d;
    const int nwin = p.nwin;
    uint8_t *hist = p.hist + static_cast<size_t>(blockIdx.x) * (2 * nwin) * H_CHUNK;
    const long long limit = p.err.limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NA; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int s = 0; s < NH; ++s) {
            mbar_init(&h_full[s], 1);
            mbar_init(&h_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 128);
            mbar_init(&uw_ready[s], 128);
            mbar_init(&uw_free[s], SWEEP_THREADS);
        }
        mbar_init(bs_ready, SWEEP_THREADS);
        mbar_init(bs_free, 2);
        mbar_init(drain, 1);
        mbar_init(&strip_full[0], 1);
        mbar_init(&strip_full[1], 1);
        fence_barrier_init();
        tma_prefetch_desc(&fmap);
        if (p.strip_tma)
            tma_prefetch_desc(&smap);
    }
    for (int e = threadIdx.x; e < RB * 16; e += blockDim.x) {
        const int r = e >> 4, b = e & 15;
        const bool in = r < nrows && b < M;
        c_s[r][b] = in ? p.C[(row0 + r) * M + b] : 0.f;
    }
    if (threadIdx.x < RB) {
        // every Delta of row r is a difference of two of its codewords: |Delta| <= max c - min c
        const int r = threadIdx.x;
        float lo = 0.f, hi = 0.f;
        if (r < nrows) {
            lo = hi = p.C[(row0 + r) * M];
            for (int b = 1; b < M; ++b) {
                lo = fminf(lo, p.C[(row0 + r) * M + b]);
                hi = fmaxf(hi, p.C[(row0 + r) * M + b]);
            }
        }
        const int tr = hi > lo ? clamp_scale(14 - ilogbf(hi - lo)) : 0;
        dsc[r] = pow2f(tr);
        dinv[r] = pow2f(-tr);
    }
    if (warp == 1)
        tmem_alloc(tmem_holder, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA and bulk copies
        // Pass T (window T's u): for each earlier window w <= T-2 that had a move, its two history
        // chunks (Delta pieces) and the F pieces F[T][chunk]; then the F pieces of window T-1's two
        // chunks (whose Delta the sweep is still producing). Then, once window T-1 is decided, its
        // Delta pieces go from shared memory to the history.
        if (lane == 0) {
            int aslot = 0, hslot = 0;
            // per slot: bit = parity of the number of fills, and whether it was ever filled
            uint32_t apar = 0u, aused = 0u, hpar = 0u, hused = 0u;
            int stored = 0, confirmed = 0;  // history chunks written / known complete
            bool ok = true;
            auto load_f = [&](int c, int T) -> bool {
                for (int pc = 0; pc < FPIECES; ++pc) {
                    if (!mbar_wait_sleep(&a_empty[aslot], ((apar >> aslot) & 1u) ^ 1u, limit, 64))
                        return false;
                    mbar_arrive_expect_tx(&a_full[aslot], A_TILE);
                    tma_load_3d(a_base + aslot * A_TILE, &fmap, &a_full[aslot], c * CH, T * WIN,
                                g * FPIECES + pc);
                    apar ^= 1u << aslot;
                    aused |= 1u << aslot;
                    aslot = (aslot + 1 == NA) ? 0 : aslot + 1;
                }
                return true;
            };
            for (int T = 1; T < nwin && ok; ++T) {
                for (int w = 0; w + 1 < T && ok; ++w) {
                    if (!wmask[w])
                        continue;
                    for (int h = 0; h < 2 && ok; ++h) {
                        const int c = 2 * w + h;
                        if (c >= confirmed) {
                            bulk_wait_all();
                            confirmed = stored;
                        }
                        if (!mbar_wait_sleep(&h_empty[hslot], ((hpar >> hslot) & 1u) ^ 1u, limit, 64)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&h_full[hslot], H_CHUNK);
                        bulk_load(h_base + hslot * H_CHUNK, hist + static_cast<size_t>(c) * H_CHUNK,
                                  H_CHUNK, &h_full[hslot]);
                        hpar ^= 1u << hslot;
                        hused |= 1u << hslot;
                        hslot = (hslot + 1 == NH) ? 0 : hslot + 1;
                        ok = load_f(c, T);
                    }
                }
                for (int h = 0; h < 2 && ok; ++h)
                    ok = load_f(2 * (T - 1) + h, T);
                if (ok && !mbar_wait_sleep(bs_ready, (T - 1) & 1, limit, 64))
                    ok = false;
                if (!ok) {
                    raise_error(p.err, kErrTimeout, 31);
                    break;
                }
                if (wmask[T - 1]) {
                    bulk_store(hist + static_cast<size_t>(2 * (T - 1)) * H_CHUNK, bs_base,
                               2 * H_CHUNK);
                    bulk_commit();
                    stored = 2 * T;
                    bulk_wait_read_all();
                }
                mbar_arrive(bs_free);
            }
            if (!ok) {
                // the last fill of slot s completed phase (fills - 1), parity = fills parity ^ 1
                for (int s = 0; s < NA; ++s)
                    if ((aused >> s) & 1u)
                        mbar_wait(&a_full[s], ((apar >> s) & 1u) ^ 1u, kDrainLimit);
                for (int s = 0; s < NH; ++s)
                    if ((hused >> s) & 1u)
                        mbar_wait(&h_full[s], ((hpar >> s) & 1u) ^ 1u, kDrainLimit);
            }
            bulk_wait_all();
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        // Accumulator T & 1 (32 TMEM columns, lane = coordinate of window T, column = row) gets
        // sum over chunks c of F[T][c] x Delta[c], three piece products of four K=16 MMAs each.
        if (lane == 0) {
            int aslot = 0, hslot = 0;
            uint32_t aph = 0u, hph = 0u, uses = 0u;  // bit per slot / accumulator: phase parity
            bool ok = true;
            for (int T = 1; T < nwin && ok; ++T) {
                const int acc = T & 1;
                if (!mbar_wait_sleep(&acc_empty[acc], ((uses >> acc) & 1u) ^ 1u, limit, 64)) {
                    raise_error(p.err, kErrTimeout, 32);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * RB);
                int n = 0;
                auto chunk = [&](uint32_t b_addr, bool math) -> bool {
                    for (int pa = 0; pa < FPIECES; ++pa) {
                        if (!mbar_wait_sleep(&a_full[aslot], (aph >> aslot) & 1u, limit, 64))
                            return false;
                        aph ^= 1u << aslot;
                        tc_fence_after();
                        if (math) {
                            const uint32_t sa = smem_u32(a_base + aslot * A_TILE);
                            // F1 x (D1 + D2) + F2 x D1: the dropped F2 x D2 is below 2^-22 of
                            // each term, the size of the pieces' own rounding
                            for (int pb = 0; pb < DPIECES - pa; ++pb) {
#pragma unroll
                                for (int kk = 0; kk < CH / 16; ++kk) {
                                    // K-major, 128-byte swizzle: 16 k = 32 bytes along the row
                                    const uint64_t ad = umma_desc_sw128(sa + kk * 32, 16, 1024);
                                    const uint64_t bd =
                                        umma_desc_sw128(b_addr + pb * H_PIECE + kk * 32, 16, 1024);
                                    umma_f16(d_tmem, ad, bd, IDESC, n > 0 ? 1u : 0u);
                                    ++n;
                                }
                            }
                        }
                        umma_commit(&a_empty[aslot]);
                        aslot = (aslot + 1 == NA) ? 0 : aslot + 1;
                    }
                    return true;
                };
                for (int w = 0; w + 1 < T && ok; ++w) {
                    if (!wmask[w])
                        continue;
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!mbar_wait_sleep(&h_full[hslot], (hph >> hslot) & 1u, limit, 64)) {
                            ok = false;
                            break;
                        }
                        hph ^= 1u << hslot;
                        ok = chunk(smem_u32(h_base + hslot * H_CHUNK), true);
                        umma_commit(&h_empty[hslot]);
                        hslot = (hslot + 1 == NH) ? 0 : hslot + 1;
                    }
                }
                if (ok && !mbar_wait_sleep(bs_ready, (T - 1) & 1, limit, 64))
                    ok = false;
                const bool mv = ok && wmask[T - 1] != 0;
                for (int h = 0; h < 2 && ok; ++h)
                    ok = chunk(smem_u32(bs_base + h * H_CHUNK), mv);
                if (!ok) {
                    raise_error(p.err, kErrTimeout, 33);
                    break;
                }
                umma_commit(bs_free);
                umma_commit(&acc_full[acc]);
                uses ^= 1u << acc;
            }
            umma_commit(drain);
            mbar_wait(drain, 0, kDrainLimit);
        }
    } else if (warp < 6) {
        // ---------------------------------------------------------------- window assembly
        // Thread = coordinate kl of the window (= TMEM lane; warp w reads lanes 32 (w % 4)..).
        // u of window T for the CTA's rows: u0 = F (c[q] - w) at the start of the sweep, plus the
        // accumulator of the moves made before the window, written to the window buffer T & 1.
        const int quarter = warp & 3;
        const int kl = quarter * 32 + lane;
        uint32_t uses = 0u, wuses = 0u;  // bit per buffer: phase parity
        bool anyw = false;
        for (int T = 0; T < nwin; ++T) {
            const int64_t k = static_cast<int64_t>(T) * WIN + kl;
            const bool kin = k < d;
            float u0[RB];
            // u of the CTA's rows at coordinate k (row-major u: a warp reads 128 contiguous bytes)
#pragma unroll
            for (int r = 0; r < RB; ++r)
                u0[r] = (kin && r < nrows) ? p.U[(row0 + r) * d + k] : 0.f;
            if (T > 0) {
                const int acc = T & 1;
                int okw = 0;
                if (lane == 0)
                    okw = (mbar_wait_sleep(bs_ready, (T - 1) & 1, limit, 64) &&
                           mbar_wait_sleep(&acc_full[acc], (uses >> acc) & 1u, limit, 64)) ? 1 : 0;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) {
                    if (lane == 0)
                        raise_error(p.err, kErrTimeout, 34);
                    break;
                }
                __syncwarp();
                tc_fence_after();
                uses ^= 1u << acc;
                anyw = anyw || wmask[T - 1] != 0;
                if (anyw) {
                    float D[RB];
                    tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                           static_cast<uint32_t>(acc * RB),
                                       D);
                    // the accumulator carries 2^fexp[k] 2^t_r
                    const float inv_fk = pow2f(kin ? -p.fexp[static_cast<int64_t>(g) * d + k] : 0);
#pragma unroll
                    for (int r = 0; r < RB; ++r)
                        u0[r] += (D[r] * inv_fk) * dinv[r];
                }
                tc_fence_before();
                mbar_arrive(&acc_empty[acc]);
            }
            const int buf = T & 1;
            int okw = 0;
            if (lane == 0)
                okw = mbar_wait_sleep(&uw_free[buf], ((wuses >> buf) & 1u) ^ 1u, limit, 64) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) {
                if (lane == 0)
                    raise_error(p.err, kErrTimeout, 35);
                break;
            }
            __syncwarp();
            wuses ^= 1u << buf;
            float *uw = uwb + buf * (RB * UW_LD);
#pragma unroll
            for (int r = 0; r < RB; ++r)
                uw[r * UW_LD + kl] = (kin && r < nrows) ? u0[r] : 0.f;
            mbar_arrive(&uw_ready[buf]);
        }
    } else {
        // ---------------------------------------------------------------- the sweep
        const int t = threadIdx.x - 6 * 32;  // 0..127
        const float *Fg = p.F + static_cast<int64_t>(g) * d * d;
        const bool vecF = (d & 3) == 0 && (reinterpret_cast<uintptr_t>(p.F) & 15u) == 0;
        uint32_t spar = 0u, sused = 0u;  // strip buffers: parity of TMA fills, ever filled
        // F rows b0..b0+31, columns wstart..wstart+127 of the group (zero outside F) -> strip buf:
        // one TMA box issued by thread LEAD (completing on strip_full[buf]) or, when F's rows are not
        // 16-byte multiples, loads by the threads tid = 0 .. nthr-1 of the caller
        auto load_strip = [&](int buf, int64_t b0, int64_t wstart, int tid, int nthr) {
            float *st = strip + buf * (BLK * WIN);
            if (p.strip_tma) {
                if (t == LEAD) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(&strip_full[buf], BLK * WIN * 4);
                    tma_load_3d(st, &smap, &strip_full[buf], static_cast<int32_t>(wstart),
                                static_cast<int32_t>(b0), g);
                    spar ^= 1u << buf;
                    sused |= 1u << buf;
                }
            } else if (vecF) {
                for (int e = tid; e < BLK * WIN / 4; e += nthr) {
                    const int r = e / (WIN / 4), c4 = e % (WIN / 4);
                    const int64_t row = b0 + r, col = wstart + 4 * c4;
                    float *dst = st + r * WIN + 4 * c4;
                    if (row < d && col < d)
                        cp_async16(dst, Fg + row * d + col);
                    else
                        *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                cp_async_commit();
            } else {
                for (int e = tid; e < BLK * WIN; e += nthr) {
                    const int r = e / WIN, c = e % WIN;
                    const int64_t row = b0 + r, col = wstart + c;
                    st[r * WIN + c] = (row < d && col < d) ? Fg[row * d + col] : 0.f;
                }
            }
        };
        uint32_t wuses = 0u;  // bit per window buffer: phase parity
        int bi = 0;
        // codes of row r at coordinates k0 + 8 s .. + 7 (task e = 4 r + s of the threads tid = 0 ..
        // nthr-1) into code buffer buf: asynchronous copies (completed with the block's F strip),
        // plain loads at a ragged end, 0 outside the problem. Readers mask the classes.
        const bool qvec = (d & 7) == 0 && (reinterpret_cast<uintptr_t>(p.Q) & 7u) == 0;
        auto fetch_codes = [&](int buf, int64_t k0, int tid, int nthr) {
            for (int e = tid; e < RB * 4; e += nthr) {
                const int r = e >> 2, s = e & 3;
                const int64_t k = k0 + 8 * s;
                uint8_t *dst = &qb2[buf][r][8 * s];
                if (r < nrows && k < d && qvec && k + 8 <= d) {
                    cp_async8(dst, p.Q + (row0 + r) * d + k);
                } else {
                    uint32_t w[2] = {0u, 0u};
                    if (r < nrows && k < d) {
                        const uint8_t *src = p.Q + (row0 + r) * d + k;
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2)
                            if (k + e2 < d)
                                w[e2 >> 2] |= static_cast<uint32_t>(src[e2]) << (8 * (e2 & 3));
                    }
                    *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
                }
            }
            cp_async_commit();
        };
        // The rest of decided block j (buffers jb, local index jlb, coordinates jb0 .. jb0+jnb-1)
        // by the threads tid = 0 .. nthr-1: task (row r, sub s) writes the row's new codes (8 of
        // them) and, for later windows, the Delta pieces in the K-major, 128-byte-swizzled operand
        // (row r, K = 32 (jlb & 1) + k within chunk jlb >> 1, sub s: the 16-byte chunk of
        // k = 8 s .. 8 s + 7); then, from kfrom on (kfrom < 0: none), the window's later
        // coordinates get u[r][k] += sum_ii Delta[ii][r] F[jb0 + ii][wstart + k] (thread = row and
        // 4 consecutive k, F read as a broadcast, ii in increasing order).
        auto finish_block = [&](int jb, int jlb, int64_t jb0, int jnb, int tid, int nthr, int kfrom,
                                int kend, float *uw, bool keep) {
            uint8_t(*qj)[BLK + 8] = qb2[jb];
            float(*dlj)[RB] = dl2[jb];
            for (int e = tid; e < RB * 4; e += nthr) {
                const int r = e >> 2, s = e & 3;
                const int64_t jr = row0 + r;
                if (r < nrows && rm2[jb][r] != 0u) {
                    if (qvec && 8 * s + 8 <= jnb) {
                        *reinterpret_cast<uint2 *>(p.Q + jr * d + jb0 + 8 * s) =
                            *reinterpret_cast<const uint2 *>(&qj[r][8 * s]);
                    } else {
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2) {
                            const int k = 8 * s + e2;
                            if (k < jnb)
                                p.Q[jr * d + jb0 + k] = qj[r][k];
                        }
                    }
                }
                if (keep) {
                    uint32_t pk[DPIECES][4];
                    const float sc = dsc[r];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float x0 = dlj[8 * s + 2 * e2][r] * sc;
                        const float x1 = dlj[8 * s + 2 * e2 + 1][r] * sc;
                        const __half a0 = __float2half_rn(x0), c0 = __float2half_rn(x1);
                        const __half a1 = __float2half_rn(x0 - __half2float(a0));
                        const __half c1 = __float2half_rn(x1 - __half2float(c0));
                        pk[0][e2] = static_cast<uint32_t>(__half_as_ushort(a0)) |
                                    (static_cast<uint32_t>(__half_as_ushort(c0)) << 16);
                        pk[1][e2] = static_cast<uint32_t>(__half_as_ushort(a1)) |
                                    (static_cast<uint32_t>(__half_as_ushort(c1)) << 16);
                    }
                    uint8_t *bs = bs_base + (jlb >> 1) * H_CHUNK + r * 128;
                    const int chunk16 = (4 * (jlb & 1) + s) ^ (r & 7);
#pragma unroll
                    for (int pc = 0; pc < DPIECES; ++pc)
                        *reinterpret_cast<uint4 *>(bs + pc * H_PIECE + chunk16 * 16) =
                            make_uint4(pk[pc][0], pk[pc][1], pk[pc][2], pk[pc][3]);
                }
            }
            const unsigned colmask = mv2[jb];
            if (colmask != 0u && kfrom >= 0 && kfrom < kend) {
                const int r = tid & 31, wq = tid >> 5, nw = nthr >> 5;
                const float *stw = strip + jb * (BLK * WIN);
                for (int k0 = kfrom + 4 * wq; k0 < kend; k0 += 4 * nw) {
                    float a0 = uw[r * UW_LD + k0], a1 = uw[r * UW_LD + k0 + 1];
                    float a2 = uw[r * UW_LD + k0 + 2], a3 = uw[r * UW_LD + k0 + 3];
#pragma unroll 4
                    for (int ii = 0; ii < BLK; ++ii) {
                        if ((colmask >> ii) & 1u) {
                            const float dr = dlj[ii][r];
                            const float4 f = *reinterpret_cast<const float4 *>(stw + ii * WIN + k0);
                            a0 = fmaf(dr, f.x, a0);
                            a1 = fmaf(dr, f.y, a1);
                            a2 = fmaf(dr, f.z, a2);
                            a3 = fmaf(dr, f.w, a3);
                        }
                    }
                    uw[r * UW_LD + k0] = a0;
                    uw[r * UW_LD + k0 + 1] = a1;
                    uw[r * UW_LD + k0 + 2] = a2;
                    uw[r * UW_LD + k0 + 3] = a3;
                }
            }
        };
        constexpr uint32_t MASK4 = 0x01010101u * static_cast<uint32_t>(M - 1);
        // warp 6 (lane = row): the row's codebook sorted, equal values in index order, and the
        // midpoints between neighbours, for the decisions of the whole sweep
        float mid[M > 1 ? M - 1 : 1];
        float sv[M];   // the sorted codebook
        if (warp == 6) {
            const int r = lane;
            for (int a = 0; a < M; ++a) {
                const float ca = c_s[r][a];
                int rank = 0;
                for (int b = 0; b < M; ++b) {
                    const float cb = c_s[r][b];
                    rank += (cb < ca || (cb == ca && b < a)) ? 1 : 0;
                }
                srt_s[r][rank] = ca;
                ord_s[r][rank] = static_cast<uint8_t>(a);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k + 1 < M; ++k)
                mid[k] = 0.5f * (srt_s[r][k] + srt_s[r][k + 1]);
#pragma unroll
            for (int k = 0; k < M; ++k)
                sv[k] = srt_s[r][k];
        }
        fetch_codes(0, 0, t, SWEEP_THREADS);
        load_strip(0, 0, 0, t, SWEEP_THREADS);
        bool failed = false;
        unsigned long long cmoves = 0ull, ctail = 0ull;  // warp 6: this lane's row's counters
        for (int T = 0; T < nwin; ++T) {
            const int64_t wstart = static_cast<int64_t>(T) * WIN;
            const int buf = T & 1;
            const bool keep = T + 1 < nwin;  // later windows need this window's Delta
            int mine = mbar_wait(&uw_ready[buf], (wuses >> buf) & 1u, limit) ? 1 : 0;
            if (mine && T >= 1 && keep)
                mine = mbar_wait(bs_free, (T - 1) & 1, limit) ? 1 : 0;
            if (!named_bar_and(SWEEP_BAR, SWEEP_THREADS, mine)) {
                if (t == 0)
                    raise_error(p.err, kErrTimeout, 36);
                break;
            }
            wuses ^= 1u << buf;
            float *uw = uwb + buf * (RB * UW_LD);
            bool wmoved = false;
            const int kend = (d - wstart < WIN) ? static_cast<int>(d - wstart) : WIN;
            const int nblk = (kend + BLK - 1) / BLK;  // blocks of this window
            for (int lb = 0; lb < nblk; ++lb, ++bi) {
                const int64_t b0 = wstart + lb * BLK;
                const int nb = (d - b0 < BLK) ? static_cast<int>(d - b0) : BLK;
                const int cb = bi & 1;  // strip, code and move buffers of this block
                int sok = 1;
                if (p.strip_tma)
                    sok = mbar_wait(&strip_full[cb], (bi >> 1) & 1, limit) ? 1 : 0;
                cp_async_wait_all();
                // strip and codes of this block complete, the previous block decided
                if (!named_bar_and(SWEEP_BAR, SWEEP_THREADS, sok)) {
                    if (t == 0)
                        raise_error(p.err, kErrTimeout, 37);
                    failed = true;
                    break;
                }
                if (lb > 0) {
                    // the previous block's moves into this block's u (thread: row t % 32 and 8
                    // coordinates; ii in increasing order, as for the later blocks)
                    const int pb = cb ^ 1;
                    const unsigned colmask = mv2[pb];
                    if (colmask != 0u) {
                        const int r = t & 31;
                        const int kb = lb * BLK + 8 * (t >> 5);
                        const float *stw = strip + pb * (BLK * WIN) + kb;
                        float a[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            a[e] = uw[r * UW_LD + kb + e];
#pragma unroll
                        for (int ii = 0; ii < BLK; ++ii) {
                            if ((colmask >> ii) & 1u) {
                                const float dr = dl2[pb][ii][r];
                                const float4 f0 = *reinterpret_cast<const float4 *>(stw + ii * WIN);
                                const float4 f1 = *reinterpret_cast<const float4 *>(stw + ii * WIN + 4);
                                a[0] = fmaf(dr, f0.x, a[0]);
                                a[1] = fmaf(dr, f0.y, a[1]);
                                a[2] = fmaf(dr, f0.z, a[2]);
                                a[3] = fmaf(dr, f0.w, a[3]);
                                a[4] = fmaf(dr, f1.x, a[4]);
                                a[5] = fmaf(dr, f1.y, a[5]);
                                a[6] = fmaf(dr, f1.z, a[6]);
                                a[7] = fmaf(dr, f1.w, a[7]);
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            uw[r * UW_LD + kb + e] = a[e];
                    }
                }
                const float *st = strip + cb * (BLK * WIN) + lb * BLK;  // st[ii * WIN + c]
                if (t < BLK) {
                    const float f = st[t * WIN + t];
                    fdg_s[t] = f;
                    finv_s[t] = f > 0.f ? __frcp_rn(f) : __int_as_float(0x7f800000);  // 1/0 -> +inf
                }
                named_bar_sync(SWEEP_BAR, SWEEP_THREADS);
                if (warp == 6) {
                    // Decisions (lane = row). With F_ii > 0, candidate a changes the objective by
                    // F_ii ((c_a - t)^2 - (cur - t)^2), t = cur - u_i / F_ii, so the best candidate
                    // is the codeword nearest to t: the number of midpoints of the sorted codebook
                    // below t gives it. Its change delta (2 u_i + delta F_ii) is then evaluated
                    // and the coordinate moves only if that is strictly negative. (F_ii = 0 gives
                    // t = -+inf, the extreme codeword, which is the best one for a linear change.)
                    const int r = lane;
                    const bool vr = r < nrows;
                    uint8_t(*qb_s)[BLK + 8] = qb2[cb];
                    // registers hold the block's u and codes; each coordinate's current value is
                    // read and its move written in shared memory
                    float ub[BLK];
                    // qw: the block's codes as decided so far; qo: the codes before the block, from
                    // which each coordinate's current value is read (no decision changes them, so
                    // those reads do not wait for the previous coordinate)
                    uint32_t qw[BLK / 4], qo[BLK / 4];
#pragma unroll
                    for (int v = 0; v < BLK / 4; ++v) {
                        qw[v] = *reinterpret_cast<const uint32_t *>(&qb_s[r][4 * v]) & MASK4;
                        qo[v] = qw[v];
                    }
#pragma unroll
                    for (int ii = 0; ii < BLK; ++ii)
                        ub[ii] = uw[r * UW_LD + lb * BLK + ii];
                    const unsigned rowmask = sweep_decide_block<M>(
                        ub, qw, qo, c_s[r], ord_s[r], finv_s, fdg_s, st, &dl2[cb][0][r], mid, sv,
                        vr, nb);
#pragma unroll
                    for (int v = 0; v < BLK / 4; ++v)
                        *reinterpret_cast<uint32_t *>(&qb_s[r][4 * v]) = qw[v];
                    rm2[cb][r] = rowmask;
                    {
                        const unsigned moved = static_cast<unsigned>(__popc(rowmask));
                        cmoves += moved;
                        ctail += static_cast<unsigned long long>(moved) *
                                     static_cast<unsigned long long>(d - b0) -
                                 bit_position_sum(rowmask);
                    }
                    const unsigned wm = __reduce_or_sync(0xffffffffu, rowmask);
                    if (lane == 0)
                        mv2[cb] = wm;
                } else {
                    // warps 7-9 while the block is decided: the rest of the previous block of this
                    // window (its codes, Delta pieces and the window's coordinates after this
                    // block), then the next block's codes and strip into the buffers it freed
                    const int ht = t - 32;
                    if (lb > 0)
                        finish_block(cb ^ 1, lb - 1, b0 - BLK, BLK, ht, SWEEP_THREADS - 32,
                                     (lb + 1) * BLK, kend, uw, keep);
                    named_bar_sync(HELP_BAR, SWEEP_THREADS - 32);
                    const int64_t nb0 = b0 + BLK;
                    if (nb0 < d) {
                        fetch_codes(cb ^ 1, nb0, ht, SWEEP_THREADS - 32);
                        load_strip(cb ^ 1, nb0, lb + 1 < NBLK ? wstart : wstart + WIN, ht,
                                   SWEEP_THREADS - 32);
                    }
                }
                named_bar_sync(SWEEP_BAR, SWEEP_THREADS);
                wmoved = wmoved || mv2[cb] != 0u;
                // the window's last block is finished before the window ends (its Delta pieces
                // feed the next windows' product)
                if (lb + 1 == nblk)
                    finish_block(cb, lb, b0, nb, t, SWEEP_THREADS, -1, kend, uw, keep);
            }
            if (failed)
                break;
            if (t == 0)
                wmask[T] = wmoved ? 1 : 0;
            if (keep) {
                fence_proxy_async_smem();
                mbar_arrive(bs_ready);
            }
            mbar_arrive(&uw_free[buf]);
        }
        if (warp == 6) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                cmoves += __shfl_xor_sync(0xffffffffu, cmoves, o);
                ctail += __shfl_xor_sync(0xffffffffu, ctail, o);
            }
            if (lane == 0 && p.counters != nullptr) {
                atomicAdd(&p.counters[0], cmoves);
                atomicAdd(&p.counters[1], ctail);
            }
        }
        cp_async_wait_all();
        // after an early exit, let the strip copies in flight land (the last fill of buffer b
        // completes phase fills - 1)
        if (p.strip_tma && t == LEAD)
            for (int b = 0; b < 2; ++b)
                if ((sused >> b) & 1u)
                    mbar_wait(&strip_full[b], ((spar >> b) & 1u) ^ 1u, kDrainLimit);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------
size_t lnq_sweep_history_bytes(int64_t d, int64_t d_out, int groups)
{
    const int64_t R = d_out / groups;
    const int64_t ctas = groups * ((R + sw::RB - 1) / sw::RB);
    const int64_t nwin = (d + sw::WIN - 1) / sw::WIN;
    return static_cast<size_t>(ctas) * 2 * nwin * sw::H_CHUNK;
}

// Tensor map over F (fp32 [groups][d][d]) for the sweep's strips: 128 x 32 (column x row) boxes, no
// swizzle, zeros outside d x d. Needs rows of 16-byte multiples (d % 4 == 0) and an aligned F.
static bool encode_f32_strips(CUtensorMap *map, const float *F, int64_t d, int groups)
{
    if ((d & 3) != 0 || (reinterpret_cast<uintptr_t>(F) & 15u) != 0)
        return false;
    auto encode = tensor_map_encoder();
    if (encode == nullptr)
        return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(d),
                          static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(d * d) * 4};
    cuuint32_t box[3] = {sw::WIN, sw::BLK, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(F), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int M>
static cudaError_t sweep_m(const CUtensorMap &map, const CUtensorMap &smap, const SwParams &p,
                           unsigned grid, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(sweep_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sw::SMEM));
    if (e != cudaSuccess)
        return e;
    KernelTimer timer("lnq_sweep", s);
    sweep_kernel<M><<<grid, sw::NUM_THREADS, sw::SMEM, s>>>(map, smap, p);
    return cudaGetLastError();
}

cudaError_t lnq_sweep(const float *F, const __half *Fh, const int32_t *fexp, int groups,
                      const float *U, const float *C, uint8_t *Q, uint8_t *hist, int64_t d,
                      int64_t d_out, int m, DeviceErr err, cudaStream_t s)
{
    CUtensorMap map;
    if (!encode_f16_pieces(&map, Fh, d, groups))
        return cudaErrorInvalidValue;
    CUtensorMap smap;
    memset(&smap, 0, sizeof(smap));
    const bool strip_tma = encode_f32_strips(&smap, F, d, groups);
    SwParams p{};
    p.strip_tma = strip_tma ? 1 : 0;
    p.F = F;
    p.U = U;
    p.C = C;
    p.Q = Q;
    p.hist = hist;
    p.fexp = fexp;
    p.d = d;
    p.d_out = d_out;
    p.rows_per_group = d_out / groups;
    p.blocks_per_group = static_cast<int>((p.rows_per_group + sw::RB - 1) / sw::RB);
    p.nwin = static_cast<int>((d + sw::WIN - 1) / sw::WIN);
    p.counters = reinterpret_cast<unsigned long long *>(err.flags) + kWsCounterWord;
    p.err = err;
    const unsigned grid = static_cast<unsigned>(p.blocks_per_group) * static_cast<unsigned>(groups);
    switch (m) {
    case 2: return sweep_m<2>(map, smap, p, grid, s);
    case 4: return sweep_m<4>(map, smap, p, grid, s);
    case 8: return sweep_m<8>(map, smap, p, grid, s);
    case 16: return sweep_m<16>(map, smap, p, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
