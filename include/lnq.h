/*
 * lnq.h -- C ABI of the B200 (sm_100a) library for the GuidedQuant + LNQ hot path.
 *
 * What it computes (source pages: "GuidedQuant" blog post on jinukkim.me, and the GuidedQuant
 * abstract on the aitopics "squeezellm" tag page):
 *
 *   1. Guided Fisher blocks -- GuidedQuant section, third equation and the sentence after it.
 *      The gradient-weighted output error ||dL/dZ (.) (XW - XW^)||_F^2 equals
 *      n * sum_j (w_j - w^_j)^T F_j (w_j - w^_j) with F_j = (1/n) X^T diag(G_:,j^2) X. The blocks
 *      are grouped and averaged within each group, which gives
 *          F_g = alpha * X^T diag(s_g) X,   s_g[t] = mean_{j in g} G[t,j]^2.
 *      Groups are contiguous, equal slices of output rows. With G == NULL every gradient is 1, and
 *      then F = alpha * X^T X, the Hessian of the plain layer-wise objective (first equation).
 *   2. LNQ -- LNQ section, both equations. Output row j gets a codebook c_j (m values) and a
 *      one-hot assignment q_j (d_in indices). These minimise
 *          J_j = (c_j[q_j] - w_j)^T F_g (c_j[q_j] - w_j)
 *      by alternating two steps: the closed-form codebook update c <- (P^T F P)^-1 P^T F w, and a
 *      coordinate-descent assignment sweep over i = 0..d_in-1 in order.
 *
 * Readings the pages leave open, and what this library does:
 *   - Initial codebook: c_q = sort(w)[floor((2q+1) d_in / (2m))]. Each weight then takes its
 *     nearest codeword, with ties going to the lower index. Every iteration starts with the
 *     codebook step.
 *   - Assignment: a coordinate moves only if the move strictly lowers J_j. Among equal best
 *     candidates, the lowest index wins.
 *   - Codebook: solved over the non-empty codewords only; empty codewords keep their value; no
 *     damping. If the Cholesky factorisation meets a non-positive pivot, the row keeps its old
 *     codebook and its row_status is set to LNQ_ROW_SINGULAR.
 *
 * Conventions for every entry point:
 *   - Pointers: every array pointer is DEVICE memory that the caller allocates and owns. The
 *     library allocates no device memory at run time. Its state between calls is a cached TMA
 *     encoder function pointer, per-kernel occupancy figures, and, for lnq_build_fisher_noalloc
 *     only, a static device array of LNQ_NOALLOC_SCRATCH_BYTES that is part of the library image
 *     (every GPU that loads the library holds it) with its device address cached per device.
 *     Calls that use that array must not overlap on the GPU.
 *   - Layout: all matrices are dense and row-major with no padding.
 *       X  [n][d_in]      bf16, passed as raw 16-bit patterns (uint16_t)
 *       G  [n][d_out]     bf16 (raw 16-bit), or NULL
 *       W  [d_out][d_in]  fp32, row j = output channel w_j
 *       F  [groups][d_in][d_in] fp32, full symmetric blocks
 *       C  [d_out][m]     fp32
 *       Q  [d_out][d_in]  uint8 codeword indices
 *   - Streams: each call enqueues its work on `stream` and returns without synchronising. A NULL
 *     stream is the legacy default stream. Results are valid once the stream has synchronised.
 *   - Workspace: `ws` is caller-owned device scratch of at least lnq_workspace_size(op, ...) bytes,
 *     aligned to 256 bytes. Two calls that share one workspace must not overlap in time.
 *   - Errors: a call returns LNQ_ERR_INVALID_ARG (bad sizes or misaligned pointers) or
 *     LNQ_ERR_WORKSPACE (ws too small, NULL or misaligned) before it launches anything.
 *     It returns LNQ_ERR_CUDA if a launch fails. Kernels never trap. Every wait inside them is
 *     bounded. A wait that gives up sets a flag in the workspace and the kernel returns early;
 *     lnq_workspace_check() reports that flag as LNQ_ERR_TIMEOUT.
 */
#ifndef LNQ_H
#define LNQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LNQ_API __attribute__((visibility("default")))
#else
#define LNQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (struct CUstream_st *); NULL is the legacy default stream. */
typedef struct CUstream_st *lnq_stream_t;

typedef enum {
    LNQ_OK = 0,
    LNQ_ERR_INVALID_ARG = 1,
    LNQ_ERR_CUDA = 2,
    LNQ_ERR_WORKSPACE = 3,
    LNQ_ERR_UNSUPPORTED = 4,
    LNQ_ERR_TIMEOUT = 5
} lnq_status;

/* Per-row outcome written to row_status by lnq_quantize_rows. */
enum { LNQ_ROW_OK = 0, LNQ_ROW_SINGULAR = 1, LNQ_ROW_NOT_PD = 2 };

/* Operation selector for lnq_workspace_size. */
typedef enum {
    LNQ_OP_BUILD_FISHER = 0,
    LNQ_OP_INIT_CODEBOOK = 1,
    LNQ_OP_QUANTIZE_ROWS = 2,
    LNQ_OP_OBJECTIVE = 3,
    LNQ_OP_GANQ_ROWS = 4
} lnq_op;

/* Bytes of device workspace the operation needs for these sizes (0 if the sizes are invalid).
 * Arguments an operation does not use are ignored. */
LNQ_API size_t lnq_workspace_size(lnq_op op, int64_t n, int64_t d_in, int64_t d_out, int groups, int m);

/* Guided Fisher blocks F_g = alpha * X^T diag(s_g) X, g = 0..groups-1 (GuidedQuant section, third
 * equation and the grouping sentence).
 *   X      [n][d_in] bf16; G [n][d_out] bf16 or NULL (all gradients 1, requires groups == 1)
 *   alpha  overall scale (1 gives X^T X for G == NULL; 1/n gives the blocks of the equation)
 *   F      out, [groups][d_in][d_in] fp32, both triangles written
 * Requirements: n >= 1; d_in >= 1 and d_in % 8 == 0 (X's rows are read by TMA, whose row
 * strides must be multiples of 16 bytes); d_out >= 1; groups >= 1 and d_out % groups == 0; X, G
 * and F 16-byte aligned.
 * Arithmetic: s_g[t] is reduced in fp32. The products run on tensor cores with fp32
 * accumulation. With G == NULL both operands are X in bf16 (exact products). With G != NULL the
 * operands are one-sided fp16 with power-of-two scales: A[t] = X[t] 2^-e_t (exact; 2^e_t is the
 * smallest power of two >= max_i |X[t][i]|) and B_g[t] = fp16(s_g[t] X[t] 2^(e_t - E_g)) (one
 * rounding, 2^-11 relative; 2^E_g bounds s_g[t] max_i X[t][i]^2 over the tokens), so that
 * F_g = alpha 2^E_g A^T B_g and every entry is within about 5e-4 sqrt(F_ii F_kk) of the exact
 * value, even for a single token. */
LNQ_API lnq_status lnq_build_fisher(const uint16_t *X, const uint16_t *G, int64_t n, int64_t d_in,
                            int64_t d_out, int groups, float alpha, float *F, void *ws,
                            size_t ws_bytes, lnq_stream_t stream);

/* Size in bytes of the static device scratch behind lnq_build_fisher_noalloc (64 MiB). */
#define LNQ_NOALLOC_SCRATCH_BYTES (64ull << 20)

/* lnq_build_fisher without a workspace argument. The pages have no counterpart: this entry point
 * is an addition of this library, for callers that cannot allocate device memory at the moment
 * they need F. Examples are a plugin with no allocator handle, code that runs inside another
 * framework's fixed memory pool, or a latency-critical path that cannot afford the implicit
 * synchronisation of cudaMalloc.
 *   Scratch: a file-scope device array of LNQ_NOALLOC_SCRATCH_BYTES inside the library. Every GPU
 *   that loads the library holds it until the process exits. The call itself allocates nothing
 *   (no cudaMalloc, no cudaFree, no allocating library routine).
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it. Make that first call before
 *   any stream capture, and call with the device that owns `stream` current. The cached address
 *   does not survive a cudaDeviceReset of that device: do not use the library across one.
 *   Errors: a bounded in-kernel wait that gives up sets the flag in the array's header, which the
 *   next call clears; read it with lnq_workspace_check(NULL, stream) after the call and before
 *   the next one (LNQ_ERR_TIMEOUT means F is incomplete).
 *   Sharing: all calls share the one array, which keeps the last call's contents. Each call
 *   clears what must start at zero and overwrites the rest, but calls that overlap on the GPU
 *   (different streams or host threads) race on the array, so serialise them.
 *   Arguments, results and requirements: as lnq_build_fisher. Returns LNQ_ERR_WORKSPACE, before
 *   touching the device, when the problem needs more than LNQ_NOALLOC_SCRATCH_BYTES of scratch
 *   (lnq_workspace_size(LNQ_OP_BUILD_FISHER, ...) bytes with G, 256 bytes without G). */
LNQ_API lnq_status lnq_build_fisher_noalloc(const uint16_t *X, const uint16_t *G, int64_t n,
                                            int64_t d_in, int64_t d_out, int groups, float alpha,
                                            float *F, lnq_stream_t stream);

/* Initial codebooks and assignments for every row (reading above).
 *   W  [d_out][d_in] fp32 in; C [d_out][m] fp32 out; Q [d_out][d_in] uint8 out
 * Requirements: m in {2, 4, 8, 16}; 1 <= d_in <= 16384; d_out >= 1. */
LNQ_API lnq_status lnq_init_codebook(const float *W, int64_t d_out, int64_t d_in, int m, float *C,
                             uint8_t *Q, void *ws, size_t ws_bytes, lnq_stream_t stream);

/* `iters` LNQ iterations (codebook step, then assignment sweep) for every row, starting from
 * (C, Q) and updating them in place (LNQ section, second equation). Row j uses
 * F[j / (d_out/groups)].
 *   J_out       [d_out] fp64 out (objective after the last sweep), or NULL
 *   row_status  [d_out] int32 out (LNQ_ROW_OK / LNQ_ROW_SINGULAR), or NULL
 * Resuming: calling with iters = a and then with iters = b gives bit-identical (C, Q) to one call
 * with iters = a + b.
 * Requirements: as lnq_init_codebook, plus groups >= 1, d_out % groups == 0, 0 <= iters. */
LNQ_API lnq_status lnq_quantize_rows(const float *F, int groups, const float *W, int64_t d_out,
                             int64_t d_in, int m, int iters, float *C, uint8_t *Q,
                             double *J_out, int32_t *row_status, void *ws, size_t ws_bytes,
                             lnq_stream_t stream);

/* LNQ with a diagonal Fisher block: `iters` iterations of the same codebook step and assignment
 * sweep as lnq_quantize_rows, with F_g = diag(Fd[g]).
 * "GuidedQuant" (jinukkim.me blog), opening list, item 2 (diagonal-Fisher methods keep only the
 * diagonal of the Fisher block); aitopics "squeezellm" tag page, SqueezeLLM abstract
 * (sensitivity-based non-uniform quantization); the blog's LNQ section iteration.
 * With a diagonal block the codebook step gives each non-empty codeword the weighted mean
 * sum f_i w_i / sum f_i of its coordinates (a non-empty class with sum f_i <= 0 makes the row
 * singular: it keeps its codebook and row_status reports it), and moves in the sweep do not
 * interact, so every coordinate takes its nearest codeword in the f_i-weighted sense (only a
 * strictly lower cost moves; the lowest index wins among equals).
 *   Fd          [groups][d_in] fp32 device, row j uses Fd[j / (d_out/groups)]
 *   W, C, Q     as lnq_quantize_rows (C, Q in/out; codes are read modulo m)
 *   J_out       [d_out] fp64 out, sum_i f_i (C[j][Q[j][i]] - W[j][i])^2, or NULL
 *   row_status  [d_out] int32 out, or NULL
 * Arithmetic: the class sums are exact integer sums of per-coordinate fixed-point terms
 * (rint(f_i w_i 2^s_w), rint(f_i 2^s_f), every term at most 2^41 for the row's scales); a class
 * whose f sum is under n_a 2^24 units is summed directly in fp64 instead. Moves are decided by
 * fp32 midpoints and confirmed by the fp64 change; objective terms in fp32, summed in fp64 in a
 * fixed order. Results are bit-identical from run to run and across any split of the iterations
 * over calls. Needs no workspace.
 * Requirements: non-NULL Fd, W, C, Q; m in {2, 4, 8, 16}; 1 <= d_in <= 16384; 1 <= d_out < 2^31;
 * groups >= 1 and d_out % groups == 0; iters >= 0. Otherwise LNQ_ERR_INVALID_ARG before any
 * device work; a launch failure is LNQ_ERR_CUDA. */
LNQ_API lnq_status lnq_quantize_rows_diag(const float *Fd, int groups, const float *W,
                                          int64_t d_out, int64_t d_in, int m, int iters, float *C,
                                          uint8_t *Q, double *J_out, int32_t *row_status,
                                          lnq_stream_t stream);

/* A GANQ-style comparison solver on the same per-row problem: `iters` iterations of the
 * codebook step of lnq_quantize_rows followed by a Cholesky / back-substitution assignment.
 * scime.ai summary of GANQ (GPU-adaptive non-uniform quantization), Approach paragraph
 * (alternating Cholesky / back-substitution index assignment and closed-form least-squares
 * codebook, batched on the GPU). Reading: F_g = L L^T with L lower (factorised once per call in
 * fp64); with r = C[j][Q[j]] - W[j], coordinates are visited from the last to the first and each
 * takes the codeword nearest to t_i = w_i - (sum_{k > i} L[k][i] r_k) / L[i][i]; no damping.
 *   F, W, C, Q, J_out  as lnq_quantize_rows (C, Q in/out; codes are read modulo m)
 *   row_status  [d_out] int32 out, or NULL: LNQ_ROW_SINGULAR as lnq_quantize_rows; LNQ_ROW_NOT_PD
 *               for rows of a group whose factorisation met a non-positive pivot (their codes are
 *               kept; the codebook step still runs)
 *   ws          lnq_workspace_size(LNQ_OP_GANQ_ROWS, 0, d_in, d_out, groups, m) bytes, 256-byte
 *               aligned (the QUANTIZE_ROWS workspace plus an fp64 and an fp32 copy of every F_g
 *               and a residual per weight).
 * Arithmetic: factorisation in fp64; the back-substituted sums in fp32 from the fp32 factor, in a
 * fixed order, so results are bit-identical from run to run.
 * Requirements and errors as lnq_quantize_rows. */
LNQ_API lnq_status lnq_ganq_rows(const float *F, int groups, const float *W, int64_t d_out,
                                 int64_t d_in, int m, int iters, float *C, uint8_t *Q,
                                 double *J_out, int32_t *row_status, void *ws, size_t ws_bytes,
                                 lnq_stream_t stream);

/* Per-row objective J[j] = r^T F_g r with r = C[j][Q[j]] - W[j] ("GuidedQuant" blog, GuidedQuant
 * section, third equation: the guided output error of row j is n r^T F_j r; LNQ section, first
 * equation, with F_g in place of X^T X). Row j uses F[j / (d_out/groups)].
 *   W, C, Q  as lnq_quantize_rows (read only); J [d_out] fp64 out
 * Arithmetic: u = F r on tensor cores (F and r as fp16 pieces, fp32 accumulation), then J = r^T u
 * with fp64 sums. Requirements and errors as lnq_quantize_rows; `ws` as for
 * LNQ_OP_OBJECTIVE. */
LNQ_API lnq_status lnq_objective(const float *F, int groups, const float *W, const float *C,
                         const uint8_t *Q, int64_t d_out, int64_t d_in, int m, double *J,
                         void *ws, size_t ws_bytes, lnq_stream_t stream);

/* Synchronises `stream`, then reads and clears the flag that a bounded in-kernel wait sets when it
 * gives up. ws == NULL checks the static scratch of lnq_build_fisher_noalloc on the current
 * device. Returns LNQ_OK, LNQ_ERR_TIMEOUT or LNQ_ERR_CUDA. */
LNQ_API lnq_status lnq_workspace_check(void *ws, lnq_stream_t stream);

/* Work counters of the assignment sweeps of the last lnq_quantize_rows call that used `ws` (LNQ
 * section, the coordinate loop): *moves = coordinates that changed codeword, summed over rows and
 * iterations; *tail = the sum over those moves of (d_in - i), i the 0-based coordinate, which is
 * the number of entries of u = F r that each move updates. Synchronises `stream`. Returns
 * LNQ_ERR_INVALID_ARG for a NULL or misaligned ws or NULL outputs. */
LNQ_API lnq_status lnq_sweep_counters(const void *ws, lnq_stream_t stream, int64_t *moves,
                                      int64_t *tail);

/* Measurement aid (no counterpart on the pages): enqueues a kernel of independent FP32 FFMA chains
 * over every SM (8 blocks of 256 threads per SM, each thread `iters` x 8 FFMAs) so that the caller
 * can time the device's FP32 lane-operation rate with CUDA events on `stream`. *lane_ops receives
 * the number of FFMAs the launch performs. sink: device memory of at least one float, written
 * never in practice (it keeps the chains live). Requirements: iters a positive multiple of 16. */
LNQ_API lnq_status lnq_fp32_probe(int64_t iters, float *sink, int64_t *lane_ops,
                                  lnq_stream_t stream);

/* ---- Consumer of (C, Q): packed codes and the lookup-table GEMV ----------------------------
 * "GuidedQuant" (jinukkim.me blog), LNQ section, last sentence (LNQ runs on SqueezeLLM's CUDA
 * kernel); aitopics "squeezellm" tag page, SqueezeLLM and GANQ abstracts (single-batch inference
 * is memory-bound; weights as low-bit indices into a lookup table).
 * Packed format (the pages fix none): bits = log2(m) in {1, 2, 3, 4}; row j is a run of
 * lnq_packed_words(d_in, bits) 32-bit words of floor(32 / bits) codes each, code i in word
 * i / floor(32 / bits) at bit (i mod floor(32 / bits)) * bits, unused bits zero. */

/* 32-bit words per packed row (0 if bits is not in 1..4 or d_in < 1). */
LNQ_API int64_t lnq_packed_words(int64_t d_in, int bits);

/* Packs Q [d_out][d_in] uint8 (device, codes < 2^bits; higher bits are dropped) into
 * P [d_out][lnq_packed_words(d_in, bits)] uint32 (device, caller-owned).
 * Requirements: bits in 1..4, d_out >= 1, d_in >= 1, non-NULL pointers; otherwise
 * LNQ_ERR_INVALID_ARG. */
LNQ_API lnq_status lnq_pack_codes(const uint8_t *Q, int64_t d_out, int64_t d_in, int bits,
                                  uint32_t *P, lnq_stream_t stream);

/* y[b][j] = sum_i x[b][i] * C[j][code(j, i)] for b < nb: nb activation vectors times the
 * quantised weights W^ = C[Q], read from the packed codes.
 *   x [nb][d_in] fp32, P packed as above, C [d_out][2^bits] fp32, y [nb][d_out] fp32 out; all
 *   device memory, caller-owned.
 * Arithmetic: fp32 products and sums in a fixed order (per row, each lane sums its words in order;
 * the 32 lanes by a fixed shuffle butterfly; the 16 warps that split d_in in order), so results
 * are bit-identical from run to run.
 * Requirements: bits in 1..4, 1 <= nb <= 8, d_out >= 1, d_in >= 1, non-NULL pointers; otherwise
 * LNQ_ERR_INVALID_ARG. */
LNQ_API lnq_status lnq_lut_gemv(const float *x, int64_t nb, const uint32_t *P, const float *C,
                                int64_t d_out, int64_t d_in, int bits, float *y,
                                lnq_stream_t stream);

/* Testing knob: upper bound, in SM clock cycles, on every in-kernel wait of later calls from this
 * process (0 makes every wait give up at once). A negative value restores the default of about
 * 2^31 cycles, roughly a second. */
LNQ_API void lnq_set_wait_limit(int64_t cycles);

/* Tracing aid: when switched on (on != 0), every kernel launch of later calls is bracketed by two
 * CUDA events on the launching stream. Off by default; events are host objects, so profiling
 * allocates no device memory. */
LNQ_API void lnq_profile_enable(int on);

/* Waits for the recorded events, then writes at most max_kernels entries: names[k] (static
 * strings owned by the library), total_ms[k] (summed device time) and launches[k]. Clears the
 * records. Returns the number of entries written. */
LNQ_API int lnq_profile_read(int max_kernels, const char **names, double *total_ms,
                             int64_t *launches);

/* Static description of a status code. */
LNQ_API const char *lnq_status_string(lnq_status status);

#ifdef __cplusplus
}
#endif

#endif /* LNQ_H */
