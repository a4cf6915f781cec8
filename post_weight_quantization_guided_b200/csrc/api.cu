// api.cu -- the extern "C" entry points declared in include/lnq.h.
//
// Host-side only: argument validation, workspace carving, TMA descriptor encoding and kernel
// launches on the caller's stream. No device memory is allocated here.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "lnq_internal.cuh"
#include "profile.cuh"

namespace lnq {

// Kernels and launchers defined in fisher.cu.
__global__ void token_stats_kernel(const __nv_bfloat16 *, const __nv_bfloat16 *, int64_t, int64_t,
                                   int64_t, int64_t, int, float *, float *, unsigned *);
__global__ void token_scales_kernel(int64_t, int64_t, int, float *, float *, const unsigned *);
cudaError_t fisher_syrk(const __nv_bfloat16 *X, const float *S, const float *M,
                        const unsigned *pimax, int64_t n, int64_t ld, int64_t d, int groups,
                        float alpha, float *F, DeviceErr err, cudaStream_t s, int num_sms);

static std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

static int device_sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return 148;
    return sms;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool valid_m(int m) { return m == 2 || m == 4 || m == 8 || m == 16; }

// Workspace layout (all offsets 256-byte aligned):
//   BUILD_FISHER:   header | S [groups][ld] f32 | M [ld] f32 | pimax [groups] u32
//                   (ld = n rounded up to a multiple of 64)
//   QUANTIZE_ROWS:  header | status [d_out] i32 | Fh [groups][2][d_in][ld] f16 (ld = d_in
//                   rounded up to a multiple of 8) | fexp [groups][d_in] i32 | rexp [d_out] i32
//                   | Sb [2 ceil(d_in / 256)][d_out][m][m] f32 (class-binned partial sums)
//                   | U [d_out][d_in] f32 (-F w) | Ur [d_out][d_in] f32 (u = F r)
//                   | sweep history [CTAs][2 ceil(d_in / 128)][2][4 KB] (Delta pieces)
//                   | right-operand image of the products [row tiles][K blocks][256][64] 16-bit
//   OBJECTIVE:      the same layout (status, Sb and U unused)
//   GANQ_ROWS:      the QUANTIZE_ROWS layout, then A [groups][d_in][d_in] f64 (the factorisation)
//                   | L [groups][d_in][d_in] f32 | 1 / L_ii [groups][d_in] f32
//                   | R [d_out][d_in] f32 (residuals) | factor status [groups] i32
//   INIT:           header
struct FisherWs {
    size_t s_off, m_off, pi_off, total;
};
static int64_t fisher_ld(int64_t n) { return (n + 63) / 64 * 64; }
static FisherWs fisher_ws(int64_t n, int groups)
{
    FisherWs w;
    const int64_t ld = fisher_ld(n);
    w.s_off = kWsHeader;
    w.m_off = align_up(w.s_off + static_cast<size_t>(groups) * ld * sizeof(float), 256);
    w.pi_off = align_up(w.m_off + static_cast<size_t>(ld) * sizeof(float), 256);
    w.total = align_up(w.pi_off + static_cast<size_t>(groups) * sizeof(unsigned), 256);
    return w;
}

struct LnqWs {
    size_t st_off, fh_off, fexp_off, rexp_off, sb_off, u_off, ur_off, hist_off, img_off, total;
};
static LnqWs lnq_ws(int64_t d_in, int64_t d_out, int groups, int m)
{
    LnqWs w;
    w.st_off = kWsHeader;
    w.fh_off = align_up(w.st_off + static_cast<size_t>(d_out) * 4, 256);
    const size_t ld = static_cast<size_t>((d_in + 7) / 8 * 8);  // fp16 piece row stride
    w.fexp_off = align_up(w.fh_off + static_cast<size_t>(groups) * 2 * d_in * ld * 2, 256);
    w.rexp_off = align_up(w.fexp_off + static_cast<size_t>(groups) * d_in * 4, 256);
    w.sb_off = align_up(w.rexp_off + static_cast<size_t>(d_out) * 4, 256);
    w.u_off = align_up(w.sb_off + lnq_binned_bytes(d_in, d_out, m), 256);
    w.ur_off = align_up(w.u_off + static_cast<size_t>(d_in) * d_out * 4, 256);
    w.hist_off = align_up(w.ur_off + static_cast<size_t>(d_in) * d_out * 4, 256);
    w.img_off = align_up(w.hist_off + lnq_sweep_history_bytes(d_in, d_out, groups), 256);
    w.total = align_up(w.img_off + lnq_vgemm_image_bytes(d_in, d_out, groups, m), 256);
    return w;
}

static LnqWorkspace carve(void *ws, const LnqWs &lay)
{
    uint8_t *b = static_cast<uint8_t *>(ws);
    LnqWorkspace w;
    w.status = reinterpret_cast<int32_t *>(b + lay.st_off);
    w.Fh = reinterpret_cast<__half *>(b + lay.fh_off);
    w.fexp = reinterpret_cast<int32_t *>(b + lay.fexp_off);
    w.rexp = reinterpret_cast<int32_t *>(b + lay.rexp_off);
    w.Sb = reinterpret_cast<float *>(b + lay.sb_off);
    w.U = reinterpret_cast<float *>(b + lay.u_off);
    w.Ur = reinterpret_cast<float *>(b + lay.ur_off);
    w.hist = b + lay.hist_off;
    w.img = reinterpret_cast<uint16_t *>(b + lay.img_off);
    return w;
}

}  // namespace lnq

using namespace lnq;

extern "C" {

const char *lnq_status_string(lnq_status s)
{
    switch (s) {
    case LNQ_OK: return "ok";
    case LNQ_ERR_INVALID_ARG: return "invalid argument";
    case LNQ_ERR_CUDA: return "CUDA error";
    case LNQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LNQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case LNQ_ERR_TIMEOUT: return "a bounded in-kernel wait gave up";
    }
    return "unknown status";
}

void lnq_set_wait_limit(int64_t cycles)
{
    g_wait_limit.store(cycles < 0 ? kDefaultWaitLimit : static_cast<long long>(cycles));
}

size_t lnq_workspace_size(lnq_op op, int64_t n, int64_t d_in, int64_t d_out, int groups, int m)
{
    (void)m;
    switch (op) {
    case LNQ_OP_BUILD_FISHER:
        if (n < 1 || d_in < 1 || groups < 1)
            return 0;
        return fisher_ws(n, groups).total;
    case LNQ_OP_QUANTIZE_ROWS:
    case LNQ_OP_OBJECTIVE:
        if (d_out < 1 || d_in < 1 || groups < 1 || !valid_m(m))
            return 0;
        return lnq_ws(d_in, d_out, groups, m).total;
    case LNQ_OP_INIT_CODEBOOK:
        return kWsHeader;
    case LNQ_OP_GANQ_ROWS:
        if (d_out < 1 || d_in < 1 || groups < 1 || !valid_m(m))
            return 0;
        return lnq_ws(d_in, d_out, groups, m).total + lnq_ganq_extra_bytes(d_in, d_out, groups);
    }
    return 0;
}

static lnq_status check_ws(void *ws, size_t ws_bytes, size_t need)
{
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < need)
        return LNQ_ERR_WORKSPACE;
    return LNQ_OK;
}

lnq_status lnq_build_fisher(const uint16_t *X, const uint16_t *G, int64_t n, int64_t d_in,
                            int64_t d_out, int groups, float alpha, float *F, void *ws,
                            size_t ws_bytes, lnq_stream_t stream)
{
    if (X == nullptr || F == nullptr || n < 1 || d_in < 1 || d_in % 8 != 0 || d_out < 1 ||
        groups < 1 || d_out % groups != 0 || !aligned16(X) || !aligned16(F) ||
        (G != nullptr && !aligned16(G)) || (G == nullptr && groups != 1) ||
        n > (int64_t(1) << 31) - 64 || d_in > (int64_t(1) << 30))
        return LNQ_ERR_INVALID_ARG;
    const FisherWs lay = fisher_ws(n, groups);
    const size_t need = (G == nullptr) ? kWsHeader : lay.total;
    lnq_status st = check_ws(ws, ws_bytes, need);
    if (st != LNQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *base = static_cast<uint8_t *>(ws);
    DeviceErr err{reinterpret_cast<uint32_t *>(base), g_wait_limit.load()};
    if (cudaMemsetAsync(base, 0, kWsHeader, s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    const __nv_bfloat16 *Xb = reinterpret_cast<const __nv_bfloat16 *>(X);
    cudaError_t e;
    if (G != nullptr) {
        float *S = reinterpret_cast<float *>(base + lay.s_off);
        float *M = reinterpret_cast<float *>(base + lay.m_off);
        unsigned *pimax = reinterpret_cast<unsigned *>(base + lay.pi_off);
        if (cudaMemsetAsync(pimax, 0, static_cast<size_t>(groups) * sizeof(unsigned), s) !=
            cudaSuccess)
            return LNQ_ERR_CUDA;
        const int threads = 256;
        {
            KernelTimer timer("token_stats", s);
            token_stats_kernel<<<static_cast<unsigned>((n * 32 + threads - 1) / threads), threads,
                                 0, s>>>(Xb, reinterpret_cast<const __nv_bfloat16 *>(G), n,
                                         fisher_ld(n), d_in, d_out, groups, S, M, pimax);
        }
        {
            KernelTimer timer("token_scales", s);
            token_scales_kernel<<<static_cast<unsigned>((fisher_ld(n) + threads - 1) / threads),
                                  threads, 0, s>>>(n, fisher_ld(n), groups, S, M, pimax);
        }
        if (cudaGetLastError() != cudaSuccess)
            return LNQ_ERR_CUDA;
        e = fisher_syrk(Xb, S, M, pimax, n, fisher_ld(n), d_in, groups, alpha, F, err, s,
                        device_sm_count());
    } else {
        e = fisher_syrk(Xb, nullptr, nullptr, nullptr, n, n, d_in, 1, alpha, F, err, s,
                        device_sm_count());
    }
    if (e == cudaErrorNotSupported)
        return LNQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

lnq_status lnq_init_codebook(const float *W, int64_t d_out, int64_t d_in, int m, float *C,
                             uint8_t *Q, void *ws, size_t ws_bytes, lnq_stream_t stream)
{
    if (W == nullptr || C == nullptr || Q == nullptr || d_out < 1 || d_in < 1 || d_in > 16384 ||
        !valid_m(m) || d_out > (int64_t(1) << 31) - 1)
        return LNQ_ERR_INVALID_ARG;
    lnq_status st = check_ws(ws, ws_bytes, kWsHeader);
    if (st != LNQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return lnq_init_launch(W, d_out, d_in, m, C, Q, s) == cudaSuccess ? LNQ_OK : LNQ_ERR_CUDA;
}

lnq_status lnq_quantize_rows(const float *F, int groups, const float *W, int64_t d_out,
                             int64_t d_in, int m, int iters, float *C, uint8_t *Q,
                             double *J_out, int32_t *row_status, void *ws, size_t ws_bytes,
                             lnq_stream_t stream)
{
    if (F == nullptr || W == nullptr || C == nullptr || Q == nullptr || groups < 1 ||
        d_out < 1 || d_out % groups != 0 || d_in < 1 || d_in > 16384 || !valid_m(m) ||
        iters < 0 || d_out > (int64_t(1) << 31) - 1)
        return LNQ_ERR_INVALID_ARG;
    const LnqWs lay = lnq_ws(d_in, d_out, groups, m);
    lnq_status st = check_ws(ws, ws_bytes, lay.total);
    if (st != LNQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const LnqWorkspace w = carve(ws, lay);
    DeviceErr err{reinterpret_cast<uint32_t *>(ws), g_wait_limit.load()};
    if (cudaMemsetAsync(ws, 0, lay.fh_off, s) != cudaSuccess)   // header and row status
        return LNQ_ERR_CUDA;
    if (lnq_iterate_launch(F, groups, W, d_out, d_in, m, iters, C, Q, J_out, w, err,
                           device_sm_count(), s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    if (row_status != nullptr &&
        cudaMemcpyAsync(row_status, w.status, static_cast<size_t>(d_out) * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return LNQ_OK;
}

lnq_status lnq_ganq_rows(const float *F, int groups, const float *W, int64_t d_out, int64_t d_in,
                         int m, int iters, float *C, uint8_t *Q, double *J_out,
                         int32_t *row_status, void *ws, size_t ws_bytes, lnq_stream_t stream)
{
    if (F == nullptr || W == nullptr || C == nullptr || Q == nullptr || groups < 1 ||
        d_out < 1 || d_out % groups != 0 || d_in < 1 || d_in > 16384 || !valid_m(m) ||
        iters < 0 || d_out > (int64_t(1) << 31) - 1)
        return LNQ_ERR_INVALID_ARG;
    const LnqWs lay = lnq_ws(d_in, d_out, groups, m);
    lnq_status st = check_ws(ws, ws_bytes, lay.total + lnq_ganq_extra_bytes(d_in, d_out, groups));
    if (st != LNQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const LnqWorkspace w = carve(ws, lay);
    DeviceErr err{reinterpret_cast<uint32_t *>(ws), g_wait_limit.load()};
    if (cudaMemsetAsync(ws, 0, lay.fh_off, s) != cudaSuccess)   // header and row status
        return LNQ_ERR_CUDA;
    if (lnq_ganq_launch(F, groups, W, d_out, d_in, m, iters, C, Q, J_out, w,
                        static_cast<uint8_t *>(ws) + lay.total, err, device_sm_count(), s) !=
        cudaSuccess)
        return LNQ_ERR_CUDA;
    if (row_status != nullptr &&
        cudaMemcpyAsync(row_status, w.status, static_cast<size_t>(d_out) * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    return LNQ_OK;
}

lnq_status lnq_quantize_rows_diag(const float *Fd, int groups, const float *W, int64_t d_out,
                                  int64_t d_in, int m, int iters, float *C, uint8_t *Q,
                                  double *J_out, int32_t *row_status, lnq_stream_t stream)
{
    if (Fd == nullptr || W == nullptr || C == nullptr || Q == nullptr || groups < 1 ||
        d_out < 1 || d_out % groups != 0 || d_in < 1 || d_in > 16384 || !valid_m(m) ||
        iters < 0 || d_out > (int64_t(1) << 31) - 1)
        return LNQ_ERR_INVALID_ARG;
    return lnq_diag_launch(Fd, groups, W, d_out, d_in, m, iters, C, Q, J_out, row_status,
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? LNQ_OK
               : LNQ_ERR_CUDA;
}

lnq_status lnq_objective(const float *F, int groups, const float *W, const float *C,
                         const uint8_t *Q, int64_t d_out, int64_t d_in, int m, double *J,
                         void *ws, size_t ws_bytes, lnq_stream_t stream)
{
    if (F == nullptr || W == nullptr || C == nullptr || Q == nullptr || J == nullptr ||
        groups < 1 || d_out < 1 || d_out % groups != 0 || d_in < 1 || d_in > 16384 ||
        !valid_m(m) || d_out > (int64_t(1) << 31) - 1)
        return LNQ_ERR_INVALID_ARG;
    const LnqWs lay = lnq_ws(d_in, d_out, groups, m);
    lnq_status st = check_ws(ws, ws_bytes, lay.total);
    if (st != LNQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const LnqWorkspace w = carve(ws, lay);
    DeviceErr err{reinterpret_cast<uint32_t *>(ws), g_wait_limit.load()};
    if (cudaMemsetAsync(ws, 0, kWsHeader, s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    // iters = 0 with J requested: only the objective pass runs (C and Q are not modified).
    return lnq_iterate_launch(F, groups, W, d_out, d_in, m, 0, const_cast<float *>(C),
                              const_cast<uint8_t *>(Q), J, w, err, device_sm_count(),
                              s) == cudaSuccess
               ? LNQ_OK
               : LNQ_ERR_CUDA;
}

int64_t lnq_packed_words(int64_t d_in, int bits)
{
    if (bits < 1 || bits > 4 || d_in < 1)
        return 0;
    return lnq_lut_words(d_in, bits);
}

lnq_status lnq_pack_codes(const uint8_t *Q, int64_t d_out, int64_t d_in, int bits, uint32_t *P,
                          lnq_stream_t stream)
{
    if (Q == nullptr || P == nullptr || bits < 1 || bits > 4 || d_out < 1 || d_in < 1)
        return LNQ_ERR_INVALID_ARG;
    return lnq_pack_launch(Q, d_out, d_in, bits, P, device_sm_count(),
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? LNQ_OK
               : LNQ_ERR_CUDA;
}

lnq_status lnq_lut_gemv(const float *x, int64_t nb, const uint32_t *P, const float *C,
                        int64_t d_out, int64_t d_in, int bits, float *y, lnq_stream_t stream)
{
    if (x == nullptr || P == nullptr || C == nullptr || y == nullptr || bits < 1 || bits > 4 ||
        nb < 1 || nb > 8 || d_out < 1 || d_in < 1)
        return LNQ_ERR_INVALID_ARG;
    return lnq_lut_gemv_launch(x, static_cast<int>(nb), P, C, d_out, d_in, bits, y,
                               device_sm_count(), reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? LNQ_OK
               : LNQ_ERR_CUDA;
}

lnq_status lnq_workspace_check(void *ws, lnq_stream_t stream)
{
    if (ws == nullptr) {
        // the static scratch of lnq_build_fisher_noalloc on the current device
        ws = noalloc_scratch_address();
        if (ws == nullptr)
            return LNQ_ERR_CUDA;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t flags[2] = {0, 0};
    if (cudaMemcpyAsync(flags, ws, sizeof(flags), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    if (flags[0] != 0u) {
        if (cudaMemsetAsync(ws, 0, sizeof(flags), s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return LNQ_ERR_CUDA;
        return LNQ_ERR_TIMEOUT;
    }
    return LNQ_OK;
}

lnq_status lnq_sweep_counters(const void *ws, lnq_stream_t stream, int64_t *moves, int64_t *tail)
{
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || moves == nullptr ||
        tail == nullptr)
        return LNQ_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned long long c[2] = {0ull, 0ull};
    if (cudaMemcpyAsync(c, static_cast<const unsigned long long *>(ws) + kWsCounterWord, sizeof(c),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return LNQ_ERR_CUDA;
    *moves = static_cast<int64_t>(c[0]);
    *tail = static_cast<int64_t>(c[1]);
    return LNQ_OK;
}

}  // extern "C"
