// lnq_internal.cuh -- declarations shared between the library's translation units (not part of
// the C ABI).
#pragma once

#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace lnq {

// cuTensorMapEncodeTiled from the driver, looked up once; nullptr if unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Device scratch of lnq_quantize_rows / lnq_objective, carved from the caller's workspace.
struct LnqWorkspace {
    int32_t *status;     // [d_out] sticky per-row status
    __half *Fh;          // [groups][2][d][ld] fp16 pieces of F, rows scaled by 2^fexp
    int32_t *fexp;       // [groups][d]
    int32_t *rexp;       // [d_out] residual scales
    uint16_t *img;       // right-operand image of the product, lnq_vgemm_image_bytes()
    float *Sb;           // class-binned partial sums of P^T F P, lnq_binned_bytes()
    float *U;            // [d_out][d] -F w per row (fixed during a call)
    float *Ur;           // [d_out][d] u = F r per row (start of each sweep; the objective)
    uint8_t *hist;       // sweep history, lnq_sweep_history_bytes()
};

// noalloc.cu: device address of the static scratch array on the current device (nullptr if it
// cannot be found)
void *noalloc_scratch_address();

// lnq.cu
cudaError_t lnq_init_launch(const float *W, int64_t d_out, int64_t d, int m, float *C,
                            uint8_t *Q, cudaStream_t s);
cudaError_t lnq_iterate_launch(const float *F, int groups, const float *W, int64_t d_out,
                               int64_t d, int m, int iters, float *C, uint8_t *Q, double *J,
                               const LnqWorkspace &w, DeviceErr err, int num_sms, cudaStream_t s);

// lnq_vgemm.cu
bool encode_f16_pieces(CUtensorMap *map, const __half *Fh, int64_t d, int groups);
cudaError_t lnq_split_f16(const float *F, int64_t d, int groups, __half *Fh, int32_t *fexp,
                          cudaStream_t s);
cudaError_t lnq_residual_scale(const uint8_t *Q, const float *W, const float *C, int64_t d,
                               int64_t d_out, int m, int32_t *rexp, cudaStream_t s);
size_t lnq_vgemm_image_bytes(int64_t d, int64_t d_out, int groups, int m);
size_t lnq_binned_bytes(int64_t d, int64_t d_out, int m);
cudaError_t lnq_vgemm(const __half *Fh, const int32_t *fexp, const int32_t *rexp, int groups,
                      const uint8_t *Q, const float *W, const float *C, float *Sb, float *U,
                      uint16_t *img, int64_t d, int64_t d_out, int m, bool residual_only,
                      DeviceErr err, int num_sms, cudaStream_t s);

// lnq_solve.cu
cudaError_t lnq_solve(const float *Sb, int nhalves, const float *U, const uint8_t *Q, float *C,
                      int32_t *status, int64_t d, int64_t d_out, int m, cudaStream_t s);
cudaError_t lnq_objective_from_u(const float *U, const float *W, const float *C,
                                 const uint8_t *Q, double *J, int64_t d, int64_t d_out, int m,
                                 cudaStream_t s);

// lnq_sweep.cu
size_t lnq_sweep_history_bytes(int64_t d, int64_t d_out, int groups);
cudaError_t lnq_sweep(const float *F, const __half *Fh, const int32_t *fexp, int groups,
                      const float *U, const float *C, uint8_t *Q, uint8_t *hist, int64_t d,
                      int64_t d_out, int m, DeviceErr err, cudaStream_t s);

// lut.cu
int64_t lnq_lut_words(int64_t d_in, int bits);
cudaError_t lnq_pack_launch(const uint8_t *Q, int64_t d_out, int64_t d_in, int bits, uint32_t *P,
                            int num_sms, cudaStream_t s);
cudaError_t lnq_lut_gemv_launch(const float *x, int nb, const uint32_t *P, const float *C,
                                int64_t d_out, int64_t d_in, int bits, float *y, int num_sms,
                                cudaStream_t s);

// ganq.cu
size_t lnq_ganq_extra_bytes(int64_t d, int64_t d_out, int groups);
cudaError_t lnq_ganq_launch(const float *F, int groups, const float *W, int64_t d_out, int64_t d,
                            int m, int iters, float *C, uint8_t *Q, double *J,
                            const LnqWorkspace &w, void *extra, DeviceErr err, int num_sms,
                            cudaStream_t s);

// lnq_diag.cu
cudaError_t lnq_diag_launch(const float *Fd, int groups, const float *W, int64_t d_out, int64_t d,
                            int m, int iters, float *C, uint8_t *Q, double *J, int32_t *status,
                            cudaStream_t s);

}  // namespace lnq
