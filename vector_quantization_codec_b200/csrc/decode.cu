// decode.cu -- QAM-W decoder (paper section 3.2): packed indices -> BF16 rows.
//
// One thread decodes one chunk of 64 columns (32 pairs) of one row:
//   unpack its 32 indices from `bits` 32-bit words (the chunk's bit range is
//   word aligned: 32 * bits bits), look each codeword up in shared memory,
//   scale pair k by sigma_k, run the inverse Hadamard butterflies (in
//   registers, then across the lanes of the block for b > 64), multiply column
//   j by r_hat * D_j / (sqrt(b) * s_j), round to BF16; the warp then writes its
//   4 KB of output with coalesced 16-byte stores.
// The kernel is bound by HBM: it reads bits/16 bytes and writes 2 bytes per
// weight.
#include <utility>

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

constexpr int kDecThreads = 256;

// x[2q], x[2q+1] = sigma_q * codeword(index q), indices extracted one by one
template <int BITS, int... Q>
__device__ __forceinline__ void gather_pairs(const uint32_t (&w)[BITS], const float2* cb,
                                             const float* sgc, int C, float (&x)[kE],
                                             std::integer_sequence<int, Q...>) {
  (
      [&] {
        const float2 cw = cb[extract_idx<BITS, Q>(w)];
        const float s = sgc[Q * C];
        x[2 * Q] = cw.x * s;
        x[2 * Q + 1] = cw.y * s;
      }(),
      ...);
}

// Per-column factors live transposed in shared memory, [position in chunk][chunk],
// so that the 32 lanes of a warp (32 consecutive chunks) read 32 consecutive
// words.  Each warp's output -- 32 chunks of 64 BF16 = 4 KB, contiguous in W_hat
// because virtual thread v owns bytes [128 v, 128 v + 128) -- is staged in a
// swizzled shared tile (16-byte unit t of lane l at slot t ^ (l & 7), no bank
// conflicts on either side) and written back with 512-byte coalesced stores.
template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* stage = reinterpret_cast<uint4*>(smem);                  // [warps][32 lanes][8]
  float2* cb = reinterpret_cast<float2*>(stage + blockDim.x * 8);
  const int P = a.d_in >> 1, C = a.d_in / kE;
  float* sgT = reinterpret_cast<float*>(cb + a.K);  // [q][c] = sigma_{32c+q}
  float* gT = sgT + P;                               // [j][c] = D/(sqrt(b) s) of column 64c+j

  // table fills: unrolled so that each thread's loads are in flight together
#pragma unroll 4
  for (int i = threadIdx.x; i < a.K; i += blockDim.x) cb[i] = a.codebook[i];
#pragma unroll 4
  for (int k = threadIdx.x; k < P; k += blockDim.x)
    sgT[(k % kQ) * C + k / kQ] = __half2float(a.sigma[k]);
  const float inv_sqrt_b = 1.0f / sqrtf((float)a.block);
#pragma unroll 4
  for (int j = threadIdx.x; j < a.d_in; j += blockDim.x) {
    const float v = inv_sqrt_b / __half2float(a.scale[j]);
    gT[(j % kE) * C + j / kE] = mask_negative(a.seed, (uint32_t)j) ? -v : v;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  uint4* wstage = stage + (threadIdx.x >> 5) * 256;
  const int64_t V = (int64_t)a.d_out * C;
  const int nb = min(a.block, kE);
  const int lanes = max(a.block / kE, 1);
  uint4* out16 = reinterpret_cast<uint4*>(a.out);
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
    float x[kE];
    gather_pairs<BITS>(w, cb, sgT + c, C, x, std::make_integer_sequence<int, kQ>{});
    fwht_reg<kE>(x, nb);
    fwht_lanes<kE>(x, lanes);

    const float rn = active ? __half2float(a.rnorm[row]) : 0.f;
#pragma unroll
    for (int t = 0; t < kE / 8; ++t) {
      uint32_t u[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 8 * t + 2 * e;
        u[e] = pack_bf16x2(x[j] * rn * gT[j * C + c], x[j + 1] * rn * gT[(j + 1) * C + c]);
      }
      wstage[lane * 8 + (t ^ (lane & 7))] = make_uint4(u[0], u[1], u[2], u[3]);
    }
    __syncwarp();
    // unit uu = 32 i + lane of this warp's 4 KB belongs to lane uu / 8, slot uu % 8
    const int64_t wbase = base + (threadIdx.x & ~31);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int uu = 32 * i + lane, owner = uu >> 3, t = uu & 7;
      if (wbase + owner < V) out16[(wbase + owner) * 8 + t] = wstage[owner * 8 + (t ^ (owner & 7))];
    }
    __syncwarp();
  }
}

size_t decode_smem(int threads, const DecodeArgs& a) {
  return (size_t)threads * 128 + (size_t)a.K * sizeof(float2) +
         (size_t)(a.d_in / 2) * sizeof(float) + (size_t)a.d_in * sizeof(float);
}

template <int BITS>
cudaError_t run_decode(const DecodeArgs& a, cudaStream_t stream) {
  // 256 threads, or 128 when the per-column tables of a very wide matrix leave
  // no room for a 32 KB staging tile within the 227 KB a CTA may use
  const int threads = decode_smem(kDecThreads, a) <= 227 * 1024 ? kDecThreads : kDecThreads / 2;
  const size_t smem = decode_smem(threads, a);
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
