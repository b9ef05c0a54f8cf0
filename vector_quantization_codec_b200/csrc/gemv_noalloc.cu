// gemv_noalloc.cu -- the fused decode-GEMV for callers that cannot allocate.
//
// qamw_decode_gemv needs a caller-provided workspace for the rotated
// activation xbar.  Some callers have no way to provide one: plugins whose
// host interface passes only input and output pointers, engines that reserve
// all free device memory up front for their own pools (so any later
// cudaMalloc fails), and latency-critical loops that must not call cudaMalloc
// or cudaFree because those calls synchronise the device.  This entry point
// keeps xbar in a fixed array in device memory instead, reserved when the
// library's device code is loaded on a GPU and held by that GPU until the
// process exits.
//
// The array's name is only a host-side stand-in in host code, never a device
// address: the host looks the real address up with cudaGetSymbolAddress (with
// the device current) and hands that pointer to the unchanged
// qamw_decode_gemv kernels.  The lookup is cached per device together with the
// CUDA context it was made in; when the device's context has been recreated
// (after cudaDeviceReset, for example) the address is looked up again, so a
// stale address is never used.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

// Room for the rotated activation: 1 MiB.  The call accepts padded batch x
// d_in / 2 <= 131072 pairs, where the batch is padded to 1, 4, 8 or 16 (e.g.
// batch 16 with d_in <= 16384, or any batch of 8 or fewer with d_in up to the
// library limit of 32768); every accepted shape's activation fits.
constexpr size_t kNoAllocPairs = 131072;
static __device__ __align__(256) float2 g_xbar_scratch[kNoAllocPairs];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The current CUDA context (driver entry point looked up once), or null.
CUcontext current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  }();
  CUcontext ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Address of g_xbar_scratch on the current device, looked up on the first call
// in each context of the device and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr || ctx == nullptr || ctx != g_scratch_ctx[dev]) {
    // the lookup makes the device's context current if no call has yet
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_xbar_scratch);
    if (err != cudaSuccess) return err;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

int padded_batch(int batch) { return batch == 1 ? 1 : (batch <= 4 ? 4 : (batch <= 8 ? 8 : 16)); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qamw

using namespace qamw;

extern "C" QAMW_API int qamw_decode_gemv_noalloc(const qamw_matrix* m, const uint16_t* d_x,
                                                 int batch, uint16_t* d_y, int32_t* d_status,
                                                 void* stream) {
  if (m == nullptr) return QAMW_ERR_INVALID;
  if (m->bits < 1 || m->bits > 11) return QAMW_ERR_INVALID;
  if (m->d_out < 0 || m->d_in <= 0 || m->d_in % kE != 0 || m->d_in > kMaxDin) return QAMW_ERR_SHAPE;
  if (m->block <= 0 || (m->block & (m->block - 1)) != 0 || m->block > 1024 || m->d_in % m->block != 0)
    return QAMW_ERR_SHAPE;
  if (m->row_bytes != qamw_row_bytes(m->d_in, m->bits)) return QAMW_ERR_INVALID;
  if (batch < 1 || batch > 16) return QAMW_ERR_INVALID;
  // the fixed scratch bounds the problem size
  if ((size_t)padded_batch(batch) * (size_t)(m->d_in / 2) > kNoAllocPairs) return QAMW_ERR_SHAPE;
  if (m->d_out == 0) return QAMW_OK;
  if (!m->packed || !m->row_norm || !m->sigma || !m->chan_scale || !m->codebook) return QAMW_ERR_INVALID;
  if (!aligned16(m->packed) || !aligned16(m->codebook)) return QAMW_ERR_ALIGN;
  if (!aligned16(m->sigma) || !aligned16(m->chan_scale)) return QAMW_ERR_ALIGN;
  if (!d_x || !d_y) return QAMW_ERR_INVALID;
  if (!aligned16(d_x)) return QAMW_ERR_ALIGN;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return QAMW_ERR_CUDA;
  const cudaError_t err = launch_decode_gemv(*m, d_x, batch, d_y, scratch, d_status,
                                             static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? QAMW_OK : QAMW_ERR_CUDA;
}
