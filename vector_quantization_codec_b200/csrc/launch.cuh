// launch.cuh -- host-side launchers of the QAM-W kernels (called by api.cu
// after argument validation) and launch-shape helpers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "qamw.h"

namespace qamw {

// Number of SMs of the current device (cached per device).
int sm_count();

// Grid for a grid-stride kernel: enough CTAs to cover `work_ctas`, at most the
// number that can be resident at once (occupancy-limited), a multiple of the
// SM count when the work allows.
int persistent_grid(const void* kernel, int threads, size_t smem, int64_t work_ctas);

// Opt a kernel into more than 48 KB of dynamic shared memory.
cudaError_t allow_smem(const void* kernel, size_t smem);

// Launch of a path kernel with programmatic stream serialisation: it may start
// while the kernel ahead of it in the stream finishes (the kernel itself waits,
// with pdl_wait, before it touches that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same for a kernel chosen at run time (args: pointers to its arguments).
inline cudaError_t launch_pdl_ptr(const void* kernel, dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kernel, args);
}

// Workspace carve-up of qamw_encode.
struct EncodeWorkspace {
  int32_t* cal_nonzero;  // [kCalCtas] non-zero rows each CTA found among rows 0..1023
                         // (the first byte of the calibration workspace)
  int32_t* n_cal;        // [1] rows used by eq. (1)
  float* cal_ext;        // [P] |z_k| sums of rows past 1023 (zero rows present)
  float* cal_partial;    // [kCalCtas][P] partial sums of |z_k|
  void* prefilter;       // prefilter table (when the matrix carries none)
};
constexpr int kCalRows = 1024;
constexpr int kCalCtas = 32;  // CTAs per matrix of eq. (1): 32 rows each
size_t calibrate_workspace_bytes(int d_out, int d_in, EncodeWorkspace* carve, void* base);
size_t calibrate_many_workspace_bytes(const qamw_matrix* ms, int n);
size_t encode_workspace_bytes(int d_out, int d_in, int bits, EncodeWorkspace* carve, void* base);

size_t train_workspace_bytes(int bits);
size_t gemv_workspace_bytes(int d_in, int batch);

cudaError_t launch_decode(const qamw_matrix& m, uint16_t* d_out_bf16, int32_t* d_status,
                          cudaStream_t stream);
cudaError_t launch_decode_many(const qamw_matrix* ms, int n, uint16_t* const* d_outs,
                               int32_t* d_status, cudaStream_t stream);
cudaError_t launch_channel_scales(const float* d_act_stat, int d_in, float alpha, uint16_t* d_scale,
                                  int32_t* d_status, cudaStream_t stream);
cudaError_t launch_calibrate(const void* d_W, int dtype, const qamw_matrix& m,
                             const EncodeWorkspace& ws, int32_t* d_status, cudaStream_t stream);
// Channel scales and eq. (1) of n matrices (workspace: calibrate_many_workspace_bytes).
cudaError_t launch_calibrate_many(const void* const* d_W, int dtype, const float* const* d_act,
                                  float alpha, const qamw_matrix* ms, int n, void* d_ws,
                                  int32_t* d_status, cudaStream_t stream);
// Normalised points of rows [row0, row0 + nrows) as float2 [nrows][d_in / 2].
cudaError_t launch_points(const void* d_W, int dtype, const qamw_matrix& m, int64_t row0,
                          int64_t nrows, float* d_points, int32_t* d_status, cudaStream_t stream);
cudaError_t launch_encode_rows(const void* d_W, int dtype, const qamw_matrix& m, int32_t* d_status,
                               unsigned long long* d_candidates, int mode, cudaStream_t stream);
cudaError_t launch_polar_codebook(int bits, float* d_codebook, cudaStream_t stream);
cudaError_t launch_scalar_codebook(int bits, float* d_codebook, cudaStream_t stream);
cudaError_t launch_encode(const void* d_W, int dtype, const float* d_act_stat, float alpha,
                          int flags, const qamw_matrix& m, const EncodeWorkspace& ws,
                          int32_t* d_status, cudaStream_t stream);
// Table of G x G cells (prefilter_grid(bits) for the encoder) for the
// codebook of 2^bits entries; d_table holds prefilter_bytes_for(G) bytes.
cudaError_t launch_build_prefilter(const float* d_codebook, int bits, int G, void* d_table,
                                   cudaStream_t stream);
cudaError_t launch_train(const float* d_samples, int64_t n, int bits, int iters,
                         float* d_codebook, double* d_distortion, void* d_ws,
                         int32_t* d_status, cudaStream_t stream);
size_t gemm_workspace_bytes(int d_out, int d_in, int ntok);
cudaError_t launch_decode_gemm(const qamw_matrix& m, const uint16_t* d_x, int ntok, uint16_t* d_y,
                               void* d_ws, int32_t* d_status, cudaStream_t stream);
cudaError_t launch_decode_gemv(const qamw_matrix& m, const uint16_t* d_x, int batch,
                               uint16_t* d_y, void* d_ws, int32_t* d_status,
                               cudaStream_t stream);
// Batch-1 products of n matrices (workspace: gemv_many_workspace_bytes).
size_t gemv_many_workspace_bytes(const qamw_matrix* ms, int n);
cudaError_t launch_decode_gemv_many(const qamw_matrix* ms, int n, const uint16_t* const* d_x,
                                    uint16_t* const* d_y, void* d_ws, int32_t* d_status,
                                    cudaStream_t stream);

}  // namespace qamw
