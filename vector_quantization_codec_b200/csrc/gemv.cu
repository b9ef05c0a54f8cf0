// gemv.cu -- fused decode + skinny product y = x W_hat^T without forming W_hat.
//
// W_hat row i = r_i * diag(1/s) R_inv yhat_i with yhat_i pair k = sigma_k c[idx_ik]
// (paper section 3.2).  R_inv = R_fwd^T, so
//   y[t][i] = r_i * sum_k < xbar_t[k], c[idx_ik] >,  xbar_t = sigma (.) R_fwd(x_t / s)
// (pair k = coordinates 2k, 2k+1).  k_rotate computes xbar once per call into
// the workspace; k_gemv streams the packed indices and gathers codewords.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

// xbar[t][k] (float2) for t < batch, zeros for batch <= t < bpad; one thread
// per (t, chunk of 64 columns).
__global__ void __launch_bounds__(256) k_rotate(const __nv_bfloat16* __restrict__ x, int batch,
                                                int bpad, int d_in, int block, uint64_t seed,
                                                const __half* __restrict__ s,
                                                const __half* __restrict__ sigma,
                                                float2* __restrict__ xbar, int32_t* status) {
  const int C = d_in / kE, P = d_in / 2;
  const int64_t V = (int64_t)bpad * C;
  const int nb = min(block, kE), lanes = max(block / kE, 1);
  const float inv_sqrt_b = 1.0f / sqrtf((float)block);
  int flags = 0;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < V;
       base += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = base + threadIdx.x;
    const bool active = v < V;
    const int64_t t = active ? v / C : 0;
    const int c = active ? (int)(v - t * C) : 0;
    const bool real = active && t < batch;
    float xv[kE];
    if (real) {
      load64(x + t * d_in + (int64_t)c * kE, xv);
#pragma unroll
      for (int j = 0; j < kE; ++j) {
        const int col = c * kE + j;
        if (!isfinite(xv[j])) flags = QAMW_STATUS_NONFINITE;
        const float q = __fdiv_rn(xv[j], __half2float(s[col]));
        xv[j] = mask_negative(seed, (uint32_t)col) ? -q : q;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kE; ++j) xv[j] = 0.f;
    }
    fwht_reg<kE>(xv, nb);
    fwht_lanes<kE>(xv, lanes);
    if (active) {
      float2* dst = xbar + t * P + (int64_t)c * kQ;
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float sg = __half2float(sigma[c * kQ + q]) * inv_sqrt_b;
        dst[q] = make_float2(xv[2 * q] * sg, xv[2 * q + 1] * sg);
      }
    }
  }
  raise_flag(status, flags);
}

// One warp per output row; lanes take the row's 32-pair chunks round robin.
template <int BITS, int B>
__global__ void __launch_bounds__(256) k_gemv(const uint8_t* __restrict__ packed, int64_t row_bytes,
                                              const __half* __restrict__ rnorm,
                                              const float2* __restrict__ codebook, int K,
                                              const float2* __restrict__ xbar, int d_out, int d_in,
                                              int batch, __nv_bfloat16* __restrict__ y) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2* cb = reinterpret_cast<float2*>(smem);
  for (int i = threadIdx.x; i < K; i += blockDim.x) cb[i] = codebook[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int C = d_in / kE, P = d_in / 2;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < d_out; row += warps) {
    float acc[B];
#pragma unroll
    for (int t = 0; t < B; ++t) acc[t] = 0.f;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + (int64_t)row * row_bytes);
    for (int c = lane; c < C; c += 32) {
      uint32_t w[BITS];
#pragma unroll
      for (int t = 0; t < BITS; ++t) w[t] = __ldg(src + (size_t)c * BITS + t);
      uint32_t idx[kQ];
      unpack32<BITS>(w, idx);
#pragma unroll
      for (int q = 0; q < kQ; q += 2) {
        const float2 c0 = cb[idx[q]], c1 = cb[idx[q + 1]];
#pragma unroll
        for (int t = 0; t < B; ++t) {
          const float4 xb = __ldg(reinterpret_cast<const float4*>(xbar + (int64_t)t * P + c * kQ + q));
          acc[t] = fmaf(xb.x, c0.x, fmaf(xb.y, c0.y, fmaf(xb.z, c1.x, fmaf(xb.w, c1.y, acc[t]))));
        }
      }
    }
#pragma unroll
    for (int t = 0; t < B; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane == 0) {
      const float rn = __half2float(rnorm[row]);
#pragma unroll
      for (int t = 0; t < B; ++t)
        if (t < batch) y[(int64_t)t * d_out + row] = __float2bfloat16_rn(acc[t] * rn);
    }
  }
}

template <int BITS, int B>
cudaError_t run_gemv(const qamw_matrix& m, int batch, const float2* xbar, uint16_t* d_y,
                     cudaStream_t stream) {
  const int threads = 256, K = 1 << m.bits;
  const size_t smem = (size_t)K * sizeof(float2);
  const void* fn = reinterpret_cast<const void*>(&k_gemv<BITS, B>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(fn, threads, smem, ((int64_t)m.d_out * 32 + threads - 1) / threads);
  k_gemv<BITS, B><<<grid, threads, smem, stream>>>(
      m.packed, m.row_bytes, reinterpret_cast<const __half*>(m.row_norm),
      reinterpret_cast<const float2*>(m.codebook), K, xbar, m.d_out, m.d_in, batch,
      reinterpret_cast<__nv_bfloat16*>(d_y));
  return cudaGetLastError();
}

template <int BITS>
cudaError_t gemv_bits(const qamw_matrix& m, int batch, const float2* xbar, uint16_t* d_y,
                      cudaStream_t stream) {
  if (batch == 1) return run_gemv<BITS, 1>(m, batch, xbar, d_y, stream);
  if (batch <= 4) return run_gemv<BITS, 4>(m, batch, xbar, d_y, stream);
  if (batch <= 8) return run_gemv<BITS, 8>(m, batch, xbar, d_y, stream);
  return run_gemv<BITS, 16>(m, batch, xbar, d_y, stream);
}

}  // namespace

size_t gemv_workspace_bytes(int d_in, int batch) {
  // xbar padded to 16 batch columns so that the widest kernel can read them
  (void)batch;
  return (size_t)16 * (size_t)(d_in / 2) * sizeof(float2);
}

cudaError_t launch_decode_gemv(const qamw_matrix& m, const uint16_t* d_x, int batch,
                               uint16_t* d_y, void* d_ws, int32_t* d_status,
                               cudaStream_t stream) {
  float2* xbar = static_cast<float2*>(d_ws);
  const int bpad = batch == 1 ? 1 : (batch <= 4 ? 4 : (batch <= 8 ? 8 : 16));
  {
    const int threads = 256;
    const int64_t V = (int64_t)bpad * (m.d_in / kE);
    const void* fn = reinterpret_cast<const void*>(&k_rotate);
    const int grid = persistent_grid(fn, threads, 0, (V + threads - 1) / threads);
    k_rotate<<<grid, threads, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(d_x), batch,
                                           bpad, m.d_in, m.block, m.mask_seed,
                                           reinterpret_cast<const __half*>(m.chan_scale),
                                           reinterpret_cast<const __half*>(m.sigma), xbar,
                                           d_status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  // The kernel runs B = 1/4/8/16 columns; columns batch..B-1 read the zeroed
  // xbar padding and are not written to y.
  switch (m.bits) {
    case 1: return gemv_bits<1>(m, batch, xbar, d_y, stream);
    case 2: return gemv_bits<2>(m, batch, xbar, d_y, stream);
    case 3: return gemv_bits<3>(m, batch, xbar, d_y, stream);
    case 4: return gemv_bits<4>(m, batch, xbar, d_y, stream);
    case 5: return gemv_bits<5>(m, batch, xbar, d_y, stream);
    case 6: return gemv_bits<6>(m, batch, xbar, d_y, stream);
    case 7: return gemv_bits<7>(m, batch, xbar, d_y, stream);
    case 8: return gemv_bits<8>(m, batch, xbar, d_y, stream);
    case 9: return gemv_bits<9>(m, batch, xbar, d_y, stream);
    case 10: return gemv_bits<10>(m, batch, xbar, d_y, stream);
    case 11: return gemv_bits<11>(m, batch, xbar, d_y, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qamw
