// api.cu -- extern "C" entry points of libqamw.so: argument checks, workspace
// carving and dispatch to the kernels.  Nothing here allocates device memory.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// Occupancy and shared-memory opt-in are per (device, kernel, shape) facts:
// computed once and cached, so that a call costs the launches and little else.
namespace {
struct LaunchKey {
  int dev;
  const void* fn;
  int threads;
  size_t smem;
  bool operator==(const LaunchKey& o) const {
    return dev == o.dev && fn == o.fn && threads == o.threads && smem == o.smem;
  }
};
struct LaunchCache {
  std::mutex mu;
  LaunchKey key[256];
  int value[256];
  int n = 0;
};
LaunchCache g_occupancy, g_smem_optin;

bool cache_get(LaunchCache& c, const LaunchKey& k, int* v) {
  std::lock_guard<std::mutex> lock(c.mu);
  for (int i = 0; i < c.n; ++i)
    if (c.key[i] == k) {
      *v = c.value[i];
      return true;
    }
  return false;
}

void cache_put(LaunchCache& c, const LaunchKey& k, int v) {
  std::lock_guard<std::mutex> lock(c.mu);
  for (int i = 0; i < c.n; ++i)
    if (c.key[i] == k) return;
  if (c.n < 256) {
    c.key[c.n] = k;
    c.value[c.n] = v;
    ++c.n;
  }
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}
}  // namespace

int persistent_grid(const void* kernel, int threads, size_t smem, int64_t work_ctas) {
  const LaunchKey k{current_device(), kernel, threads, smem};
  int per_sm = 0;
  if (!cache_get(g_occupancy, k, &per_sm)) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
            cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    cache_put(g_occupancy, k, per_sm);
  }
  const int64_t resident = (int64_t)per_sm * sm_count();
  int64_t g = work_ctas < resident ? work_ctas : resident;
  return (int)(g < 1 ? 1 : g);
}

cudaError_t allow_smem(const void* kernel, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  // the attribute is a maximum: one call with the largest size seen so far
  const LaunchKey k{current_device(), kernel, 0, 0};
  int have = 0;
  if (cache_get(g_smem_optin, k, &have) && (size_t)have >= smem) return cudaSuccess;
  const cudaError_t err =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) {
    std::lock_guard<std::mutex> lock(g_smem_optin.mu);
    bool found = false;
    for (int i = 0; i < g_smem_optin.n; ++i)
      if (g_smem_optin.key[i] == k) {
        if (g_smem_optin.value[i] < (int)smem) g_smem_optin.value[i] = (int)smem;
        found = true;
      }
    if (!found && g_smem_optin.n < 256) {
      g_smem_optin.key[g_smem_optin.n] = k;
      g_smem_optin.value[g_smem_optin.n] = (int)smem;
      ++g_smem_optin.n;
    }
  }
  return err;
}

}  // namespace qamw

using namespace qamw;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Shape rules shared by every matrix call.
int check_shape(int d_out, int d_in, int block, int bits) {
  if (bits < 1 || bits > 11) return QAMW_ERR_INVALID;
  if (d_out < 0 || d_in <= 0 || d_in % kE != 0 || d_in > kMaxDin) return QAMW_ERR_SHAPE;
  if (!pow2(block) || block > 1024 || d_in % block != 0) return QAMW_ERR_SHAPE;
  return QAMW_OK;
}

int check_matrix(const qamw_matrix* m, bool need_outputs) {
  if (m == nullptr) return QAMW_ERR_INVALID;
  int rc = check_shape(m->d_out, m->d_in, m->block, m->bits);
  if (rc != QAMW_OK) return rc;
  if (m->row_bytes != qamw_row_bytes(m->d_in, m->bits)) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!m->packed || !m->row_norm || !m->sigma || !m->chan_scale || !m->codebook)
    return QAMW_ERR_INVALID;
  if (!aligned16(m->packed) || !aligned16(m->codebook)) return QAMW_ERR_ALIGN;
  if (!aligned16(m->sigma) || !aligned16(m->chan_scale)) return QAMW_ERR_ALIGN;
  if (m->prefilter && !aligned16(m->prefilter)) return QAMW_ERR_ALIGN;
  (void)need_outputs;
  return QAMW_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? QAMW_OK : QAMW_ERR_CUDA; }

}  // namespace

extern "C" {

int64_t qamw_row_bytes(int d_in, int bits) {
  if (d_in <= 0 || bits < 1 || bits > 11) return 0;
  const int64_t nbits = (int64_t)(d_in / 2) * bits;
  return ((nbits + 127) / 128) * 16;
}

int qamw_default_block(int d_in) {
  if (d_in <= 0) return 0;
  int b = 1;
  while (b < 1024 && d_in % (2 * b) == 0) b *= 2;
  return b;
}

double qamw_bits_per_weight(int d_in, int bits) {
  if (d_in <= 0) return 0.0;
  return bits / 2.0 + 16.0 / (double)d_in;
}

size_t qamw_prefilter_bytes(int bits) {
  if (bits < 1 || bits > 11) return 0;
  return prefilter_bytes_for(prefilter_grid(bits));
}

size_t qamw_workspace_bytes(int op, int d_out, int d_in, int bits, int batch) {
  if (bits < 1 || bits > 11) return 0;
  switch (op) {
    case QAMW_OP_TRAIN:
      return train_workspace_bytes(bits);
    case QAMW_OP_ENCODE:
      if (d_out < 0 || d_in <= 0 || d_in % kE || d_in > kMaxDin) return 0;
      return encode_workspace_bytes(d_out, d_in, bits, nullptr, nullptr);
    case QAMW_OP_CALIBRATE:
      if (d_out < 0 || d_in <= 0 || d_in % kE || d_in > kMaxDin) return 0;
      return calibrate_workspace_bytes(d_out, d_in, nullptr, nullptr);
    case QAMW_OP_GEMV:
      if (d_in <= 0 || d_in % kE || d_in > kMaxDin || batch < 1 || batch > 16) return 0;
      return gemv_workspace_bytes(d_in, batch);
    case QAMW_OP_GEMM:
      if (d_out < 0 || d_in <= 0 || d_in % kE || d_in > kMaxDin || batch < 1 || batch > kMaxTokens)
        return 0;
      return gemm_workspace_bytes(d_out, d_in, batch);
    default:
      return 0;
  }
}

const char* qamw_status_string(int code) {
  switch (code) {
    case QAMW_OK: return "ok";
    case QAMW_ERR_INVALID: return "invalid argument";
    case QAMW_ERR_SHAPE: return "unsupported shape (d_in a multiple of 64 up to 32768; block a power of two <= 1024 dividing d_in)";
    case QAMW_ERR_ALIGN: return "buffer not 16-byte aligned";
    case QAMW_ERR_WORKSPACE: return "workspace missing or too small";
    case QAMW_ERR_CUDA: return "CUDA launch or runtime error";
    case QAMW_STATUS_NONFINITE: return "non-finite input";
    case QAMW_STATUS_RANGE: return "binary16 range exceeded";
    case QAMW_STATUS_BAD_STAT: return "activation statistic not positive and finite";
    case QAMW_STATUS_TIMEOUT: return "a bounded wait for an asynchronous copy gave up";
    default: return code > 0 ? "several status flags" : "unknown error";
  }
}

int qamw_train_codebook(const float* d_samples, int64_t n, int bits, int iters, float* d_codebook,
                        double* d_distortion, void* d_workspace, size_t ws_bytes,
                        int32_t* d_status, void* stream) {
  if (bits < 1 || bits > 11 || iters < 0 || !d_samples || !d_codebook) return QAMW_ERR_INVALID;
  if (n < ((int64_t)1 << bits)) return QAMW_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(d_samples) & 7u) != 0) return QAMW_ERR_ALIGN;
  if (!aligned16(d_codebook)) return QAMW_ERR_ALIGN;
  if (!d_workspace || ws_bytes < train_workspace_bytes(bits)) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_train(d_samples, n, bits, iters, d_codebook, d_distortion, d_workspace,
                              d_status, static_cast<cudaStream_t>(stream)));
}

int qamw_build_prefilter(const float* d_codebook, int bits, void* d_table, size_t table_bytes,
                         void* stream) {
  if (bits < 1 || bits > 11 || !d_codebook || !d_table) return QAMW_ERR_INVALID;
  if (!aligned16(d_codebook) || !aligned16(d_table)) return QAMW_ERR_ALIGN;
  if (table_bytes < prefilter_bytes_for(prefilter_grid(bits))) return QAMW_ERR_WORKSPACE;
  return cuda_rc(launch_build_prefilter(d_codebook, bits, prefilter_grid(bits), d_table,
                                        static_cast<cudaStream_t>(stream)));
}

int qamw_encode(const void* d_W, int dtype, const float* d_act_stat, float alpha, int flags,
                const qamw_matrix* m, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                void* stream) {
  int rc = check_matrix(m, true);
  if (rc != QAMW_OK) return rc;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (flags & ~(QAMW_SIGMA_GIVEN | QAMW_SCALES_GIVEN | QAMW_POLAR | QAMW_SCALAR))
    return QAMW_ERR_INVALID;
  if ((flags & QAMW_POLAR) && (flags & QAMW_SCALAR)) return QAMW_ERR_INVALID;
  if ((flags & QAMW_SCALAR) && m->bits % 2 != 0) return QAMW_ERR_INVALID;
  if (!std::isfinite(alpha)) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W) return QAMW_ERR_INVALID;
  if (!aligned16(d_W) || !aligned16(m->chan_scale)) return QAMW_ERR_ALIGN;
  const size_t need = encode_workspace_bytes(m->d_out, m->d_in, m->bits, nullptr, nullptr);
  if (!d_workspace || ws_bytes < need) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  EncodeWorkspace ws;
  encode_workspace_bytes(m->d_out, m->d_in, m->bits, &ws, d_workspace);
  return cuda_rc(launch_encode(d_W, dtype, d_act_stat, alpha, flags, *m, ws, d_status,
                               static_cast<cudaStream_t>(stream)));
}

int qamw_channel_scales(const float* d_act_stat, int d_in, float alpha, uint16_t* d_scale,
                        int32_t* d_status, void* stream) {
  if (d_in <= 0 || d_in % kE != 0 || d_in > kMaxDin) return QAMW_ERR_SHAPE;
  if (!d_scale || !std::isfinite(alpha)) return QAMW_ERR_INVALID;
  return cuda_rc(launch_channel_scales(d_act_stat, d_in, alpha, d_scale, d_status,
                                       static_cast<cudaStream_t>(stream)));
}

int qamw_calibrate_sigma(const void* d_W, int dtype, const qamw_matrix* m, void* d_workspace,
                         size_t ws_bytes, int32_t* d_status, void* stream) {
  int rc = check_matrix(m, true);
  if (rc != QAMW_OK) return rc;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W) return QAMW_ERR_INVALID;
  if (!aligned16(d_W) || !aligned16(m->chan_scale)) return QAMW_ERR_ALIGN;
  const size_t need = calibrate_workspace_bytes(m->d_out, m->d_in, nullptr, nullptr);
  if (!d_workspace || ws_bytes < need) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  EncodeWorkspace ws;
  calibrate_workspace_bytes(m->d_out, m->d_in, &ws, d_workspace);
  return cuda_rc(launch_calibrate(d_W, dtype, *m, ws, d_status, static_cast<cudaStream_t>(stream)));
}

size_t qamw_calibrate_many_workspace_bytes(const qamw_matrix* ms, int n) {
  if (n <= 0 || !ms) return 0;
  for (int i = 0; i < n; ++i)
    if (ms[i].d_in <= 0 || ms[i].d_in % kE || ms[i].d_in > kMaxDin) return 0;
  return calibrate_many_workspace_bytes(ms, n);
}

int qamw_calibrate_many(const void* const* d_W, int dtype, const float* const* d_act_stat,
                        float alpha, const qamw_matrix* ms, int n, void* d_workspace,
                        size_t ws_bytes, int32_t* d_status, void* stream) {
  if (n < 0 || (n > 0 && (!ms || !d_W))) return QAMW_ERR_INVALID;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (!std::isfinite(alpha)) return QAMW_ERR_INVALID;
  if (n == 0) return QAMW_OK;
  for (int i = 0; i < n; ++i) {
    const int rc = check_matrix(&ms[i], true);
    if (rc != QAMW_OK) return rc;
    if (ms[i].d_out == 0) return QAMW_ERR_SHAPE;
    if (!d_W[i]) return QAMW_ERR_INVALID;
    if (!aligned16(d_W[i])) return QAMW_ERR_ALIGN;
  }
  const size_t need = calibrate_many_workspace_bytes(ms, n);
  if (!d_workspace || ws_bytes < need) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_calibrate_many(d_W, dtype, d_act_stat, alpha, ms, n, d_workspace, d_status,
                                       static_cast<cudaStream_t>(stream)));
}

int qamw_encode_rows(const void* d_W, int dtype, const qamw_matrix* m, uint64_t* d_candidates,
                     int32_t* d_status, void* stream) {
  int rc = check_matrix(m, true);
  if (rc != QAMW_OK) return rc;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W) return QAMW_ERR_INVALID;
  if (!aligned16(d_W)) return QAMW_ERR_ALIGN;
  if (d_candidates && (reinterpret_cast<uintptr_t>(d_candidates) & 7u)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_encode_rows(d_W, dtype, *m, d_status,
                                    reinterpret_cast<unsigned long long*>(d_candidates), kJointMode,
                                    static_cast<cudaStream_t>(stream)));
}

int qamw_normalised_pairs(const void* d_W, int dtype, const qamw_matrix* m, int64_t row0,
                          int64_t nrows, float* d_points, int32_t* d_status, void* stream) {
  int rc = check_matrix(m, false);
  if (rc != QAMW_OK) return rc;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (row0 < 0 || nrows < 0 || row0 + nrows > m->d_out) return QAMW_ERR_SHAPE;
  if (nrows == 0) return QAMW_OK;
  if (!d_W || !d_points || !m->sigma || !m->chan_scale) return QAMW_ERR_INVALID;
  if (!aligned16(d_W) || !aligned16(d_points)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_points(d_W, dtype, *m, row0, nrows, d_points, d_status,
                               static_cast<cudaStream_t>(stream)));
}

int qamw_encode_rows_polar(const void* d_W, int dtype, const qamw_matrix* m, int32_t* d_status,
                           void* stream) {
  int rc = check_matrix(m, true);
  if (rc != QAMW_OK) return rc;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W) return QAMW_ERR_INVALID;
  if (!aligned16(d_W)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_encode_rows(d_W, dtype, *m, d_status, nullptr, kPolarMode,
                                    static_cast<cudaStream_t>(stream)));
}

int qamw_encode_rows_scalar(const void* d_W, int dtype, const qamw_matrix* m, int32_t* d_status,
                            void* stream) {
  int rc = check_matrix(m, true);
  if (rc != QAMW_OK) return rc;
  if (m->bits % 2 != 0) return QAMW_ERR_INVALID;
  if (dtype != QAMW_DTYPE_F32 && dtype != QAMW_DTYPE_BF16) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W) return QAMW_ERR_INVALID;
  if (!aligned16(d_W)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_encode_rows(d_W, dtype, *m, d_status, nullptr, kScalarMode,
                                    static_cast<cudaStream_t>(stream)));
}

int qamw_scalar_codebook(int bits, float* d_codebook, void* stream) {
  if (bits < 2 || bits > 10 || bits % 2 != 0 || !d_codebook) return QAMW_ERR_INVALID;
  if (!aligned16(d_codebook)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_scalar_codebook(bits, d_codebook, static_cast<cudaStream_t>(stream)));
}

int qamw_polar_codebook(int bits, float* d_codebook, void* stream) {
  if (bits < 1 || bits > 11 || !d_codebook) return QAMW_ERR_INVALID;
  if (!aligned16(d_codebook)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_polar_codebook(bits, d_codebook, static_cast<cudaStream_t>(stream)));
}

int qamw_decode(const qamw_matrix* m, uint16_t* d_W_out, int32_t* d_status, void* stream) {
  int rc = check_matrix(m, false);
  if (rc != QAMW_OK) return rc;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_W_out) return QAMW_ERR_INVALID;
  if (!aligned16(d_W_out)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_decode(*m, d_W_out, d_status, static_cast<cudaStream_t>(stream)));
}

int qamw_decode_many(const qamw_matrix* ms, int n, uint16_t* const* d_W_out, int32_t* d_status,
                     void* stream) {
  if (n < 0 || (n > 0 && (!ms || !d_W_out))) return QAMW_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    const int rc = check_matrix(&ms[i], false);
    if (rc != QAMW_OK) return rc;
    if (ms[i].d_out == 0) continue;
    if (!d_W_out[i]) return QAMW_ERR_INVALID;
    if (!aligned16(d_W_out[i])) return QAMW_ERR_ALIGN;
  }
  if (n == 0) return QAMW_OK;
  return cuda_rc(launch_decode_many(ms, n, d_W_out, d_status, static_cast<cudaStream_t>(stream)));
}

int qamw_decode_gemv(const qamw_matrix* m, const uint16_t* d_x, int batch, uint16_t* d_y,
                     void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream) {
  int rc = check_matrix(m, false);
  if (rc != QAMW_OK) return rc;
  if (batch < 1 || batch > 16) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_x || !d_y) return QAMW_ERR_INVALID;
  if (!aligned16(d_x)) return QAMW_ERR_ALIGN;
  if (!d_workspace || ws_bytes < gemv_workspace_bytes(m->d_in, batch)) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_decode_gemv(*m, d_x, batch, d_y, d_workspace, d_status,
                                    static_cast<cudaStream_t>(stream)));
}

size_t qamw_decode_gemv_many_workspace_bytes(const qamw_matrix* ms, int n) {
  if (n <= 0 || !ms) return 0;
  return gemv_many_workspace_bytes(ms, n);
}

int qamw_decode_gemv_many(const qamw_matrix* ms, int n, const uint16_t* const* d_x,
                          uint16_t* const* d_y, void* d_workspace, size_t ws_bytes,
                          int32_t* d_status, void* stream) {
  if (n < 0 || (n > 0 && (!ms || !d_x || !d_y))) return QAMW_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    const int rc = check_matrix(&ms[i], false);
    if (rc != QAMW_OK) return rc;
    if (ms[i].d_out == 0) continue;
    if (!d_x[i] || !d_y[i]) return QAMW_ERR_INVALID;
    if (!aligned16(d_x[i])) return QAMW_ERR_ALIGN;
  }
  if (n == 0) return QAMW_OK;
  const size_t need = gemv_many_workspace_bytes(ms, n);
  if (need == 0) return QAMW_OK;
  if (!d_workspace || ws_bytes < need) return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_decode_gemv_many(ms, n, d_x, d_y, d_workspace, d_status,
                                         static_cast<cudaStream_t>(stream)));
}

int qamw_decode_gemm(const qamw_matrix* m, const uint16_t* d_x, int ntok, uint16_t* d_y,
                     void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream) {
  int rc = check_matrix(m, false);
  if (rc != QAMW_OK) return rc;
  if (ntok < 1 || ntok > kMaxTokens) return QAMW_ERR_INVALID;
  if (m->d_out == 0) return QAMW_OK;
  if (!d_x || !d_y) return QAMW_ERR_INVALID;
  if (!aligned16(d_x)) return QAMW_ERR_ALIGN;
  if (!d_workspace || ws_bytes < gemm_workspace_bytes(m->d_out, m->d_in, ntok))
    return QAMW_ERR_WORKSPACE;
  if (!aligned16(d_workspace)) return QAMW_ERR_ALIGN;
  return cuda_rc(launch_decode_gemm(*m, d_x, ntok, d_y, d_workspace, d_status,
                                    static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
