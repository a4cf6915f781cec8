// lnq_diag.cu -- LNQ with a diagonal Fisher block (the SqueezeLLM-style objective) on sm_100a.
//
// Source: "GuidedQuant" (jinukkim.me blog), opening list, item 2 (diagonal-Fisher methods weight
// the errors by end-loss gradients but keep only the diagonal of the Fisher block), the aitopics
// "squeezellm" tag page, SqueezeLLM abstract (sensitivity-based non-uniform quantization), and
// the blog's LNQ section iteration, applied to F = diag(f). With a diagonal
// block the iteration separates by coordinate:
//   codebook    c_a = sum_{i: q_i = a} f_i w_i / sum_{i: q_i = a} f_i   (the normal equations
//               P^T diag(f) P c = P^T diag(f) w are diagonal), over non-empty codewords; a class
//               whose weights f_i are all 0 is a zero pivot: the row keeps its codebook and is
//               flagged singular, as in the full solve;
//   assignment  moving coordinate i from c_q to c_a changes the objective by
//               f_i ((c_a - w_i)^2 - (c_q - w_i)^2) and changes no other coordinate's term, so
//               every coordinate takes its best codeword at once (lowest index among equals,
//               only a strictly negative change moves).
// diag_lnq_kernel: one CTA of 128 threads per row; the row's weights and codes stay in shared
// memory for all iterations.
//   class sums  kept as exact integers in a fixed-point form of the row: the term of coordinate i
//               is rint(f_i w_i 2^s_w) and rint(f_i 2^s_f), with 2^s_w and 2^s_f chosen from
//               exponent bounds of the row's largest |f_i w_i| and |f_i| (within a factor 4; the
//               largest fp32 product bounds the first) so that every term is at most 2^41 (rounding of a term: 2^-42 of the largest).
//               Integer sums do not depend on the order of the additions, so they are built once
//               by shared-memory atomics and then updated only for the coordinates that move
//               (minus the terms at the old class, plus at the new), and every iteration still
//               sees exactly the sums of its own assignment: results are bit-identical from run to
//               run and across any split of the iterations over calls. The sums are split over 32
//               slots per class, coordinate i always in slot (i / 4) mod 32, the lane that owns
//               its quad: the atomics of one warp instruction then touch distinct banks, and every
//               slot holds the sum of its own members (at most 512 of them). A slot keeps each sum
//               as two 32-bit limbs, the low 21 bits and the rest of the term (|rest| <= 2^20),
//               so that native 32-bit shared atomics add them and no limb leaves its range;
//   codebook    the slots are summed per class (one warp per limb, a transposing butterfly of
//               shuffles), then one warp forms c_a = (S_w[a] 2^-s_w) / (S_f[a] 2^-s_f) for every
//               non-empty class. Where S_f[a] is below n_a 2^24 (the class's mean f_i under 2^-17
//               of the row's largest, where the fixed-point error could pass 2^-25 relative; also
//               every class with no f_i > 0) the warp sums that class directly in fp64 over the
//               row instead. If some non-empty class has sum f_i <= 0 the row is singular and
//               keeps its codebook. Then the codebook sorted by value (equal values in index
//               order), the midpoints between neighbours and, per class, the open interval of w in
//               which it is the nearest codeword;
//   assignment  for f_i > 0 the change f_i ((c_a - w_i)^2 - (c_q - w_i)^2) orders the codewords
//               like the plain distances, so a coordinate strictly inside its current class's
//               interval stays (most of them, a few instructions each). The others (and f_i < 0)
//               go to a per-warp queue that full warps drain: the nearest codeword by a binary
//               search of the midpoints (the first of a run of equal values holds the lowest
//               index), taken only if the change evaluated in fp64 is strictly negative; f_i < 0
//               compares every codeword's fp64 change; f_i = 0 never moves (every change is 0);
//   objective   sum_i f_i r_i^2, each term in fp32 (relative error below 2^-21), the sum in fp64,
//               in the last pass, per thread in a data-fixed order, then a fixed tree.
// Near-ties: the midpoints are rounded to fp32, so a coordinate within rounding of a midpoint may
// keep or take the neighbour whose cost differs from the best by about f_i |c_a - c_b| ulp(w_i).
#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

constexpr int kDiagThreads = 128;
constexpr int kDiagWarps = kDiagThreads / 32;
constexpr int kDiagQueue = 32 + 4 * 32;   // a drain leaves < 32; one quad step adds <= 4 * 32
constexpr int kLimbs = 5;                 // f w low, f w rest, f low, f rest, count
constexpr int kNoExponent = -100000;      // exponent bound of a zero

template <int M>
struct DiagShared {
    int lim[kLimbs][M][32];                 // per limb, class and slot
    long long tot[kLimbs][M];               // per limb and class: the sum over the slots
    float cb[M];                            // codebook
    float srt[M];                           // codebook sorted by value
    float mids[M];                          // midpoints of neighbours in srt, mids[M-1] = +inf
    float2 keep[M];                         // per class: the open interval of w in which it stays
    uint8_t first_idx[M];                   // per sorted position: the lowest index of its value
    uint16_t queue[kDiagWarps][kDiagQueue]; // coordinates waiting for the full assignment
    double red[kDiagWarps];
    int ered[3][kDiagWarps];
    double scale_w, scale_f;                // 2^s_w, 2^s_f
    int flag;
};

__device__ __forceinline__ float f4_at(const float4 &v, int u)
{
    return u == 0 ? v.x : (u == 1 ? v.y : (u == 2 ? v.z : v.w));
}

// e with |x| < 2^e (subnormals bounded by 2^-126), kNoExponent for x = 0
__device__ __forceinline__ int diag_exponent(float x)
{
    const int biased = (__float_as_int(x) >> 23) & 0xff;
    return x == 0.f ? kNoExponent : max(biased, 1) - 126;
}

// 2^(41 - e) for the bound |x| < 2^e of the row's largest term, so that every term scales to at
// most 2^41 (1 when every term is 0). e lies in [-251, 259], 41 - e well inside the double
// exponent range.
__device__ __forceinline__ double diag_scale(int e)
{
    if (e == kNoExponent)
        return 1.0;
    return __longlong_as_double(static_cast<long long>(41 - e + 1023) << 52);
}

// Adds or removes coordinate i = (fi, wi) at class q (scale_w, scale_f: the row's 2^s_w, 2^s_f,
// read once by the caller).
template <int M>
__device__ __forceinline__ void diag_class_add(DiagShared<M> &sh, int i, int q, float fi,
                                               float wi, bool remove, double scale_w,
                                               double scale_f)
{
    // exact products in fp64, scaled by powers of two (exact), rounded to integers
    const long long tw = __double2ll_rn(static_cast<double>(fi) * static_cast<double>(wi) *
                                        scale_w);
    const long long tf = __double2ll_rn(static_cast<double>(fi) * scale_f);
    const int sg = remove ? -1 : 1;
    const int slot = (i >> 2) & 31;
    atomicAdd(&sh.lim[0][q][slot], sg * static_cast<int>(tw & 0x1fffff));
    atomicAdd(&sh.lim[1][q][slot], sg * static_cast<int>(tw >> 21));
    atomicAdd(&sh.lim[2][q][slot], sg * static_cast<int>(tf & 0x1fffff));
    atomicAdd(&sh.lim[3][q][slot], sg * static_cast<int>(tf >> 21));
    atomicAdd(&sh.lim[4][q][slot], sg);
}

// The full assignment of one coordinate with f_i != 0 (the queued ones).
template <int M>
__device__ __forceinline__ int diag_assign_full(const DiagShared<M> &sh, float fi, float wi, int q)
{
    const double dw = wi, cur = sh.cb[q];
    if (fi > 0.f) {
        int pos = 0;
#pragma unroll
        for (int step = M / 2; step > 0; step >>= 1)
            if (wi > sh.mids[pos + step - 1])
                pos += step;
        const double ca = sh.srt[pos];
        return (ca - dw) * (ca - dw) < (cur - dw) * (cur - dw) ? sh.first_idx[pos] : q;
    }
    const double fd = fi;
    double best = 0.0;
    int ba = q;
#pragma unroll
    for (int a = 0; a < M; ++a) {
        const double ca = sh.cb[a];
        const double delta = fd * ((ca - dw) * (ca - dw) - (cur - dw) * (cur - dw));
        if (delta < best) {
            best = delta;
            ba = a;
        }
    }
    return ba;
}

// f_i r_i^2 in fp32 (relative error below 2^-21), widened for the fp64 sum
__device__ __forceinline__ double diag_cost(float c, float fi, float wi)
{
    const float r = c - wi;
    return static_cast<double>(fi * (r * r));
}

// Processes the queue entries [lo, hi) of this warp, one per lane.
template <int M, bool kObjective>
__device__ __forceinline__ void diag_drain(DiagShared<M> &sh, float *ws, uint8_t *qs,
                                           const float *__restrict__ f, int warp, int lane,
                                           int lo, int hi, double &jr)
{
    __syncwarp();
    if (lo + lane < hi) {
        const int i = sh.queue[warp][lo + lane];
        const float wi = ws[i], fi = __ldg(f + i);
        const int q = qs[i];
        const int a = diag_assign_full<M>(sh, fi, wi, q);
        if (a != q) {
            const double sw = sh.scale_w, sf = sh.scale_f;
            qs[i] = static_cast<uint8_t>(a);
            diag_class_add<M>(sh, i, q, fi, wi, true, sw, sf);
            diag_class_add<M>(sh, i, a, fi, wi, false, sw, sf);
        }
        if (kObjective)
            jr += diag_cost(sh.cb[a], fi, wi);
    }
    __syncwarp();
}

// f[4k .. 4k+3], zero past d (kVec: d % 4 == 0 and f 16-byte aligned, so a quad is whole)
template <bool kVec>
__device__ __forceinline__ float4 diag_f4(const float *__restrict__ f, int k, int d)
{
    const int i0 = 4 * k;
    if (kVec)
        return i0 < d ? __ldg(reinterpret_cast<const float4 *>(f) + k)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v;
    v.x = i0 < d ? __ldg(f + i0) : 0.f;
    v.y = i0 + 1 < d ? __ldg(f + i0 + 1) : 0.f;
    v.z = i0 + 2 < d ? __ldg(f + i0 + 2) : 0.f;
    v.w = i0 + 3 < d ? __ldg(f + i0 + 3) : 0.f;
    return v;
}

// One assignment pass over the row (kObjective: the last one, which also sums the objective).
// Lanes past the row see f = 0, which never moves and adds nothing.
template <int M, bool kObjective, bool kVec>
__device__ __forceinline__ double diag_assign_pass(DiagShared<M> &sh, float *ws, uint8_t *qs,
                                                  const float *__restrict__ f, int d)
{
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const unsigned lt = (1u << lane) - 1u;
    const int nq = (d + 3) / 4;
    int qc = 0;                     // warp-uniform queue length
    double jr = 0.0;
    // the quad of the next step is loaded before this one is tested (a drain only touches the
    // coordinates this warp has already tested, never the quad loaded ahead)
    float4 wn = make_float4(0.f, 0.f, 0.f, 0.f), fn = wn;
    uint32_t qn = 0u;
    if (warp * 32 + lane < nq) {
        wn = reinterpret_cast<const float4 *>(ws)[warp * 32 + lane];
        qn = reinterpret_cast<const uint32_t *>(qs)[warp * 32 + lane];
    }
    fn = diag_f4<kVec>(f, warp * 32 + lane, d);
    for (int k0 = warp * 32; k0 < nq; k0 += kDiagThreads) {
        const float4 wv = wn, fv = fn;
        const uint32_t qv = qn;
        {
            const int kx = k0 + kDiagThreads + lane;
            const bool xin = kx < nq;
            wn = xin ? reinterpret_cast<const float4 *>(ws)[kx] : make_float4(0.f, 0.f, 0.f, 0.f);
            qn = xin ? reinterpret_cast<const uint32_t *>(qs)[kx] : 0u;
            fn = diag_f4<kVec>(f, kx, d);
        }
        const int k = k0 + lane;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float fi = f4_at(fv, u), wi = f4_at(wv, u);
            const int q = (qv >> (8 * u)) & 0xffu;
            const float2 kp = sh.keep[q];
            const bool stay = fi == 0.f || (fi > 0.f && wi > kp.x && wi < kp.y);
            if (kObjective && stay && fi != 0.f)
                jr += diag_cost(sh.cb[q], fi, wi);
            const unsigned mask = __ballot_sync(0xffffffffu, !stay);
            if (mask) {
                if (!stay)
                    sh.queue[warp][qc + __popc(mask & lt)] = static_cast<uint16_t>(4 * k + u);
                qc += __popc(mask);
            }
        }
        while (qc >= 32) {
            diag_drain<M, kObjective>(sh, ws, qs, f, warp, lane, qc - 32, qc, jr);
            qc -= 32;
        }
    }
    if (qc > 0)
        diag_drain<M, kObjective>(sh, ws, qs, f, warp, lane, 0, qc, jr);
    return jr;
}

// v[c] of every lane summed over the 32 lanes: a butterfly that halves the vector at each step,
// so that lane l ends with the sum for class l / (32 / M). Integer sums: exact in any order.
template <int M>
__device__ __forceinline__ long long diag_transpose_sum(long long (&v)[M], int lane)
{
#pragma unroll
    for (int n = M / 2, o = 16; n >= 1; n >>= 1, o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int c = 0; c < n; ++c) {
            const long long send = upper ? v[c] : v[c + n];
            const long long keep = upper ? v[c + n] : v[c];
            v[c] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int o = 16 / M; o >= 1; o >>= 1)
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    return v[0];
}

// Slot sums per limb and class (warp w takes limbs w, w + 4, ...); the caller puts barriers
// around it.
template <int M>
__device__ __forceinline__ void diag_slot_sums(DiagShared<M> &sh, int warp, int lane)
{
    for (int x = warp; x < kLimbs; x += kDiagWarps) {
        long long v[M];
#pragma unroll
        for (int c = 0; c < M; ++c)
            v[c] = sh.lim[x][c][lane];
        const long long s = diag_transpose_sum<M>(v, lane);
        if ((lane & (32 / M - 1)) == 0)
            sh.tot[x][lane / (32 / M)] = s;
    }
}

// The codebook step from the class sums, then the tables of the assignment (warp 0; the caller
// puts barriers around it).
template <int M>
__device__ __forceinline__ void diag_codebook(DiagShared<M> &sh, const float *ws,
                                              const uint8_t *qs, const float *__restrict__ f,
                                              int d, int lane)
{
    const int c = lane < M ? lane : 0;
    const long long sw = sh.tot[1][c] * (1ll << 21) + sh.tot[0][c];
    const long long sf = sh.tot[3][c] * (1ll << 21) + sh.tot[2][c];
    const long long n_a = sh.tot[4][c];
    const bool mine = lane < M && n_a > 0;
    double csw = static_cast<double>(sw) / sh.scale_w;
    double csf = static_cast<double>(sf) / sh.scale_f;
    // classes whose fixed-point f sum is too coarse: direct fp64 sums over the row, in a fixed
    // order (lane-strided, then a fixed tree)
    unsigned need = __ballot_sync(0xffffffffu, mine && !(sf >= (n_a << 24)));
    while (need) {
        const int a = __ffs(need) - 1;
        need &= need - 1;
        double xw = 0.0, xf = 0.0;
        for (int i = lane; i < d; i += 32) {
            if (qs[i] == a) {
                const double fi = __ldg(f + i);
                xw += fi * static_cast<double>(ws[i]);
                xf += fi;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            xw += __shfl_xor_sync(0xffffffffu, xw, o);
            xf += __shfl_xor_sync(0xffffffffu, xf, o);
        }
        if (lane == a) {
            csw = xw;
            csf = xf;
        }
    }
    const bool bad = mine && !(csf > 0.0);
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0)
            sh.flag = 1;
    } else if (mine) {
        sh.cb[lane] = static_cast<float>(csw / csf);
    }
    __syncwarp();
    int rank = 0;
    if (lane < M) {
        const float ca = sh.cb[lane];
#pragma unroll
        for (int b = 0; b < M; ++b) {
            const float cv = sh.cb[b];
            rank += (cv < ca || (cv == ca && b < lane)) ? 1 : 0;
        }
        sh.srt[rank] = ca;
    }
    __syncwarp();
    const float inf = __int_as_float(0x7f800000);
    if (lane < M) {
        sh.mids[lane] = lane + 1 < M ? 0.5f * (sh.srt[lane] + sh.srt[lane + 1]) : inf;
        const float v = sh.srt[lane];
        int lowest = 0;
#pragma unroll
        for (int b = M - 1; b >= 0; --b)
            if (sh.cb[b] == v)
                lowest = b;
        sh.first_idx[lane] = static_cast<uint8_t>(lowest);
    }
    __syncwarp();
    if (lane < M)
        sh.keep[lane] = make_float2(rank > 0 ? sh.mids[rank - 1] : -inf, sh.mids[rank]);
}

// kVec: d % 4 == 0, W and Fd 16-byte aligned and Q 4-byte aligned (rows as whole quads).
template <int M, bool kVec>
__global__ void __launch_bounds__(kDiagThreads, M == 16 ? 6 : 8)
    diag_lnq_kernel(const float *__restrict__ Fd, const float *__restrict__ W, int d,
                    int64_t rows_per_group, int iters, float *__restrict__ C,
                    uint8_t *__restrict__ Q, double *__restrict__ J, int32_t *__restrict__ status)
{
    __shared__ DiagShared<M> sh;
    extern __shared__ __align__(16) uint8_t dsm[];
    const int dp = (d + 15) / 16 * 16;
    float *ws = reinterpret_cast<float *>(dsm);          // [dp], zero past d
    uint8_t *qs = dsm + static_cast<size_t>(dp) * 4;     // [dp], zero past d
    const int64_t j = blockIdx.x;
    const float *f = Fd + (j / rows_per_group) * d;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    // the row into shared memory (each thread issues the loads of four quads before it uses
    // them), with the row's largest |f w| (as fp32 products), |f| and |w|
    constexpr int kBatch = 4;
    float mfw = 0.f, mf = 0.f, mw = 0.f;
    for (int k0 = t; k0 < dp / 4; k0 += kBatch * kDiagThreads) {
        float4 wv[kBatch], fv[kBatch];
        uint32_t qv[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int k = k0 + b * kDiagThreads, i0 = 4 * k;
            wv[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            qv[b] = 0u;
            if (i0 < d) {
                if (kVec) {
                    wv[b] = __ldg(reinterpret_cast<const float4 *>(W + j * d) + k);
                    qv[b] = __ldg(reinterpret_cast<const uint32_t *>(Q + j * d) + k);
                } else {
                    float w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        w[u] = i0 + u < d ? __ldg(W + j * d + i0 + u) : 0.f;
                        qv[b] |= i0 + u < d
                                     ? static_cast<uint32_t>(__ldg(Q + j * d + i0 + u)) << (8 * u)
                                     : 0u;
                    }
                    wv[b] = make_float4(w[0], w[1], w[2], w[3]);
                }
            }
            fv[b] = diag_f4<kVec>(f, k, d);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int k = k0 + b * kDiagThreads;
            if (k < dp / 4) {
                reinterpret_cast<float4 *>(ws)[k] = wv[b];
                reinterpret_cast<uint32_t *>(qs)[k] = qv[b] & (0x01010101u * (M - 1));
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float af = fabsf(f4_at(fv[b], u)), aw = fabsf(f4_at(wv[b], u));
                    mf = fmaxf(mf, af);
                    mw = fmaxf(mw, aw);
                    mfw = fmaxf(mfw, af * aw);
                }
            }
        }
    }
    // non-negative floats order like their bit patterns
    const int bfw = __reduce_max_sync(0xffffffffu, __float_as_int(mfw));
    const int bf = __reduce_max_sync(0xffffffffu, __float_as_int(mf));
    const int bw = __reduce_max_sync(0xffffffffu, __float_as_int(mw));
    if (lane == 0) {
        sh.ered[0][warp] = bfw;
        sh.ered[1][warp] = bf;
        sh.ered[2][warp] = bw;
    }
    for (int e = t; e < kLimbs * M * 32; e += kDiagThreads)
        (&sh.lim[0][0][0])[e] = 0;
    if (t < M)
        sh.cb[t] = C[j * M + t];
    __syncthreads();
    if (t == 0) {
        int bfw_ = 0, bf_ = 0, bw_ = 0;
        for (int w = 0; w < kDiagWarps; ++w) {
            bfw_ = max(bfw_, sh.ered[0][w]);
            bf_ = max(bf_, sh.ered[1][w]);
            bw_ = max(bw_, sh.ered[2][w]);
        }
        const float xfw = __int_as_float(bfw_), xf = __int_as_float(bf_), xw = __int_as_float(bw_);
        const int ef = diag_exponent(xf), ew = diag_exponent(xw);
        // |f w| < 2^e: from the largest fp32 product (one more for its rounding) where that is
        // a normal number, else from the bounds of |f| and |w| (products that overflow or
        // underflow fp32)
        int efw = kNoExponent;
        if (ef != kNoExponent && ew != kNoExponent)
            efw = (xfw >= 1.17549435e-38f && xfw <= 3.40282347e38f) ? diag_exponent(xfw) + 1
                                                                    : ef + ew;
        sh.scale_w = diag_scale(efw);
        sh.scale_f = diag_scale(ef);
        sh.flag = 0;
    }
    __syncthreads();
    double jr = 0.0;
    if (iters == 0) {
        for (int i = t; i < d; i += kDiagThreads)
            jr += diag_cost(sh.cb[qs[i]], __ldg(f + i), ws[i]);
    } else {
        // the class sums of the starting codes (thread t takes quads t, t + 128, ...: slot = lane)
        //  (the next quad's f is loaded before this one is added)
        const double sw = sh.scale_w, sf = sh.scale_f;
        float4 fn = diag_f4<kVec>(f, t, d);
        for (int k = t; k < (d + 3) / 4; k += kDiagThreads) {
            const float4 fv = fn;
            fn = diag_f4<kVec>(f, k + kDiagThreads, d);
            const float4 wv = reinterpret_cast<const float4 *>(ws)[k];
            const uint32_t qv = reinterpret_cast<const uint32_t *>(qs)[k];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (4 * k + u < d)
                    diag_class_add<M>(sh, 4 * k + u, (qv >> (8 * u)) & 0xffu, f4_at(fv, u),
                                      f4_at(wv, u), false, sw, sf);
        }
        for (int it = 0; it < iters; ++it) {
            __syncthreads();
            diag_slot_sums<M>(sh, warp, lane);
            __syncthreads();
            if (warp == 0)
                diag_codebook<M>(sh, ws, qs, f, d, lane);
            __syncthreads();
            if (it + 1 < iters)
                diag_assign_pass<M, false, kVec>(sh, ws, qs, f, d);
            else
                jr = diag_assign_pass<M, true, kVec>(sh, ws, qs, f, d);
        }
    }
    __syncthreads();
    // results: codebook, codes, objective sum_i f_i (c[q_i] - w_i)^2
    if (t < M)
        C[j * M + t] = sh.cb[t];
    if (kVec) {
        uint32_t *q4 = reinterpret_cast<uint32_t *>(Q + j * d);
        for (int k = t; k < d / 4; k += kDiagThreads)
            q4[k] = reinterpret_cast<const uint32_t *>(qs)[k];
    } else {
        for (int i = t; i < d; i += kDiagThreads)
            Q[j * d + i] = qs[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        jr += __shfl_xor_sync(0xffffffffu, jr, o);
    if (lane == 0)
        sh.red[warp] = jr;
    __syncthreads();
    if (t == 0) {
        double sum = 0.0;
#pragma unroll
        for (int w = 0; w < kDiagWarps; ++w)
            sum += sh.red[w];
        if (J != nullptr)
            J[j] = sum;
        if (status != nullptr)
            status[j] = sh.flag ? LNQ_ROW_SINGULAR : LNQ_ROW_OK;
    }
}

template <int M, bool kVec>
static cudaError_t diag_mv(const float *Fd, const float *W, int64_t d_out, int64_t d,
                           int64_t rows_per_group, int iters, float *C, uint8_t *Q, double *J,
                           int32_t *status, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>((d + 15) / 16 * 16) * 5;
    cudaError_t e = cudaFuncSetAttribute(diag_lnq_kernel<M, kVec>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    KernelTimer timer("lnq_diag", s);
    diag_lnq_kernel<M, kVec><<<static_cast<unsigned>(d_out), kDiagThreads, smem, s>>>(
        Fd, W, static_cast<int>(d), rows_per_group, iters, C, Q, J, status);
    return cudaGetLastError();
}

template <int M>
static cudaError_t diag_m(const float *Fd, const float *W, int64_t d_out, int64_t d,
                          int64_t rows_per_group, int iters, float *C, uint8_t *Q, double *J,
                          int32_t *status, cudaStream_t s)
{
    const bool vec = d % 4 == 0 && (reinterpret_cast<uintptr_t>(W) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(Fd) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(Q) & 3u) == 0;
    return vec ? diag_mv<M, true>(Fd, W, d_out, d, rows_per_group, iters, C, Q, J, status, s)
               : diag_mv<M, false>(Fd, W, d_out, d, rows_per_group, iters, C, Q, J, status, s);
}

cudaError_t lnq_diag_launch(const float *Fd, int groups, const float *W, int64_t d_out, int64_t d,
                            int m, int iters, float *C, uint8_t *Q, double *J, int32_t *status,
                            cudaStream_t s)
{
    const int64_t R = d_out / groups;
    switch (m) {
    case 2: return diag_m<2>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 4: return diag_m<4>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 8: return diag_m<8>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    case 16: return diag_m<16>(Fd, W, d_out, d, R, iters, C, Q, J, status, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lnq
