// decode.cu -- QAM-W decoder (paper section 3.2): packed indices -> BF16 rows.
//
// One thread decodes one chunk of 64 columns (32 pairs) of one row:
//   unpack its 32 indices from `bits` 32-bit words (the chunk's bit range is
//   word aligned: 32 * bits bits), look each codeword up in shared memory,
//   scale pair k by sigma_k, run the inverse Hadamard butterflies (in
//   registers, then across the lanes of the block for b > 64), multiply column
//   j by r_hat * D_j / (sqrt(b) * s_j), round to BF16 and store 128 bytes.
// The kernel is bound by HBM: it reads bits/16 bytes and writes 2 bytes per
// weight.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

struct DecodeArgs {
  const uint8_t* packed;
  const __half* rnorm;
  const __half* sigma;
  const __half* scale;
  const float2* codebook;
  __nv_bfloat16* out;
  int64_t row_bytes;
  int d_out, d_in, block, K;
  uint64_t seed;
};

template <int BITS>
__global__ void __launch_bounds__(256) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2* cb = reinterpret_cast<float2*>(smem);
  float* sg = reinterpret_cast<float*>(cb + a.K);
  const int P = a.d_in >> 1;
  float* g = sg + P;  // D_j / (sqrt(b) s_j)

  for (int i = threadIdx.x; i < a.K; i += blockDim.x) cb[i] = a.codebook[i];
  for (int k = threadIdx.x; k < P; k += blockDim.x) sg[k] = __half2float(a.sigma[k]);
  const float inv_sqrt_b = 1.0f / sqrtf((float)a.block);
  for (int j = threadIdx.x; j < a.d_in; j += blockDim.x) {
    const float v = inv_sqrt_b / __half2float(a.scale[j]);
    g[j] = mask_negative(a.seed, (uint32_t)j) ? -v : v;
  }
  __syncthreads();

  const int C = a.d_in / kE;
  const int64_t V = (int64_t)a.d_out * C;
  const int nb = min(a.block, kE);
  const int lanes = max(a.block / kE, 1);
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < V;
       base += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = base + threadIdx.x;
    const bool active = v < V;
    const int64_t row = active ? v / C : 0;
    const int c = active ? (int)(v - row * C) : 0;

    uint32_t w[BITS];
    const uint32_t* src =
        reinterpret_cast<const uint32_t*>(a.packed + row * a.row_bytes) + (size_t)c * BITS;
#pragma unroll
    for (int t = 0; t < BITS; ++t) w[t] = active ? __ldg(src + t) : 0u;
    uint32_t idx[kQ];
    unpack32<BITS>(w, idx);

    float x[kE];
    const float* sgc = sg + c * kQ;
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      const float2 cw = cb[idx[q]];
      const float s = sgc[q];
      x[2 * q] = cw.x * s;
      x[2 * q + 1] = cw.y * s;
    }
    fwht_reg<kE>(x, nb);
    fwht_lanes<kE>(x, lanes);

    if (active) {
      const float rn = __half2float(a.rnorm[row]);
      const float* gc = g + c * kE;
      uint4* dst = reinterpret_cast<uint4*>(a.out + row * a.d_in + (int64_t)c * kE);
#pragma unroll
      for (int t = 0; t < kE / 8; ++t) {
        uint32_t u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * t + 2 * e;
          u[e] = pack_bf16x2(x[j] * rn * gc[j], x[j + 1] * rn * gc[j + 1]);
        }
        dst[t] = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
  }
}

template <int BITS>
cudaError_t run_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int threads = 256;
  const size_t smem = (size_t)a.K * sizeof(float2) + (size_t)(a.d_in / 2) * sizeof(float) +
                      (size_t)a.d_in * sizeof(float);
  const void* fn = reinterpret_cast<const void*>(&k_decode<BITS>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int64_t V = (int64_t)a.d_out * (a.d_in / kE);
  const int grid = persistent_grid(fn, threads, smem, (V + threads - 1) / threads);
  k_decode<BITS><<<grid, threads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const qamw_matrix& m, uint16_t* d_out, int32_t* d_status,
                          cudaStream_t stream) {
  (void)d_status;
  DecodeArgs a;
  a.packed = m.packed;
  a.rnorm = reinterpret_cast<const __half*>(m.row_norm);
  a.sigma = reinterpret_cast<const __half*>(m.sigma);
  a.scale = reinterpret_cast<const __half*>(m.chan_scale);
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.out = reinterpret_cast<__nv_bfloat16*>(d_out);
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.d_in = m.d_in;
  a.block = m.block;
  a.K = 1 << m.bits;
  a.seed = m.mask_seed;
  switch (m.bits) {
    case 1: return run_decode<1>(a, stream);
    case 2: return run_decode<2>(a, stream);
    case 3: return run_decode<3>(a, stream);
    case 4: return run_decode<4>(a, stream);
    case 5: return run_decode<5>(a, stream);
    case 6: return run_decode<6>(a, stream);
    case 7: return run_decode<7>(a, stream);
    case 8: return run_decode<8>(a, stream);
    case 9: return run_decode<9>(a, stream);
    case 10: return run_decode<10>(a, stream);
    case 11: return run_decode<11>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qamw
