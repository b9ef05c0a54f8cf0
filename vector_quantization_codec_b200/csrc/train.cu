// train.cu -- Lloyd iterations for the joint 2D codebook on samples of the unit
// circular Gaussian (paper section 3.6 eq. 2).
//
// Per iteration:
//   prefilter: the exact nearest-codeword table of the current codebook
//              (prefilter.cu), so that each sample scores a few codewords
//              instead of K; the assignment equals the exhaustive fp32 search;
//   k_assign : every sample -> nearest codeword (fp32, lowest index on ties);
//              cell sums of x, y and of the squared distance are accumulated
//              as 64-bit integers in units of 2^-28, first in shared memory
//              then in global memory.  Integer addition is associative, so
//              the sums -- and the trained codebook -- are bitwise
//              reproducible whatever order the atomics land in.
//   k_update : c_j = sum_j / count_j (fp64 division, rounded to fp32); an empty
//              cell keeps its codeword; distortion[it] = sum d^2 / n; the
//              accumulators are cleared for the next iteration.
// The initial codebook is the first K samples.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

constexpr float kFix = 268435456.0f;  // 2^28
constexpr double kInvFix = 1.0 / 268435456.0;
// Coordinates are bounded by 2^10, so a cell sum stays below 2^63 for up to 2^25
// samples (2^10 * 2^28 * 2^25); draws of N(0, I_2) never come near the bound.
constexpr float kMaxCoord = 1024.0f;

struct TrainAccum {
  unsigned long long* sx;  // [K] two's-complement int64
  unsigned long long* sy;  // [K]
  unsigned long long* cnt; // [K]
  unsigned long long* dsum;  // [1]
  unsigned long long* nvalid;  // [1]
};

__global__ void k_init(const float2* __restrict__ samples, int K, float2* __restrict__ cb) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < K) cb[j] = samples[j];
}

__global__ void __launch_bounds__(512) k_assign(const float2* __restrict__ samples, int64_t n,
                                                const float2* __restrict__ cb, int K,
                                                const void* __restrict__ table, TrainAccum acc,
                                                int32_t* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2* cb2 = reinterpret_cast<float2*>(smem);
  unsigned long long* ssx = reinterpret_cast<unsigned long long*>(cb2 + K);
  unsigned long long* ssy = ssx + K;
  unsigned int* scnt = reinterpret_cast<unsigned int*>(ssy + K);
  __shared__ unsigned long long sd, sn;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    cb2[j] = cb[j];
    ssx[j] = 0ull;
    ssy[j] = 0ull;
    scnt[j] = 0u;
  }
  if (threadIdx.x == 0) {
    sd = 0ull;
    sn = 0ull;
  }
  PrefilterView pf;
  if (table != nullptr) {
    pf = prefilter_view(table, K);
  } else {
    pf.G = 0;
    pf.Gf = 0.f;
    pf.R = 0.f;
    pf.inv_h = 0.f;
  }
  __syncthreads();
  int flags = 0;
  unsigned long long my_d = 0ull, my_n = 0ull;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n;
       t += (int64_t)gridDim.x * blockDim.x) {
    const float2 p = samples[t];
    if (!isfinite(p.x) || !isfinite(p.y)) {
      flags |= QAMW_STATUS_NONFINITE;
      continue;
    }
    if (fabsf(p.x) >= kMaxCoord || fabsf(p.y) >= kMaxCoord) {
      flags |= QAMW_STATUS_RANGE;
      continue;
    }
    unsigned scored = 0;
    const int j = nearest_pf2(p.x, p.y, cb2, K, pf, scored, false);
    const float dx = p.x - cb2[j].x, dy = p.y - cb2[j].y;
    const float d = fmaf(dx, dx, dy * dy);
    atomicAdd(&ssx[j], (unsigned long long)__float2ll_rn(p.x * kFix));
    atomicAdd(&ssy[j], (unsigned long long)__float2ll_rn(p.y * kFix));
    atomicAdd(&scnt[j], 1u);
    my_d += (unsigned long long)__float2ll_rn(d * kFix);
    my_n += 1ull;
  }
  atomicAdd(&sd, my_d);
  atomicAdd(&sn, my_n);
  raise_flag(status, flags);
  __syncthreads();
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    if (scnt[j]) {
      atomicAdd(&acc.sx[j], ssx[j]);
      atomicAdd(&acc.sy[j], ssy[j]);
      atomicAdd(&acc.cnt[j], (unsigned long long)scnt[j]);
    }
  }
  if (threadIdx.x == 0) {
    atomicAdd(acc.dsum, sd);
    atomicAdd(acc.nvalid, sn);
  }
}

__global__ void k_update(float2* __restrict__ cb, int K, TrainAccum acc, double* distortion,
                         int it) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < K) {
    const unsigned long long c = acc.cnt[j];
    if (c > 0ull) {
      const double sx = (double)(long long)acc.sx[j] * kInvFix;
      const double sy = (double)(long long)acc.sy[j] * kInvFix;
      cb[j] = make_float2((float)(sx / (double)c), (float)(sy / (double)c));
    }
    acc.sx[j] = 0ull;
    acc.sy[j] = 0ull;
    acc.cnt[j] = 0ull;
  }
  if (j == 0) {
    const unsigned long long nv = *acc.nvalid;
    if (distortion) distortion[it] = nv ? (double)(long long)*acc.dsum * kInvFix / (double)nv : 0.0;
    *acc.dsum = 0ull;
    *acc.nvalid = 0ull;
  }
}

__global__ void k_zero_u64(unsigned long long* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0ull;
}

}  // namespace

size_t train_workspace_bytes(int bits) {
  const size_t K = (size_t)1 << bits;
  const size_t acc = ((3 * K + 2) * sizeof(unsigned long long) + 255) & ~(size_t)255;
  return acc + prefilter_bytes_for(prefilter_grid_train(bits));
}

cudaError_t launch_train(const float* d_samples, int64_t n, int bits, int iters, float* d_codebook,
                         double* d_distortion, void* d_ws, int32_t* d_status,
                         cudaStream_t stream) {
  const int K = 1 << bits;
  const float2* samples = reinterpret_cast<const float2*>(d_samples);
  float2* cb = reinterpret_cast<float2*>(d_codebook);
  unsigned long long* w = static_cast<unsigned long long*>(d_ws);
  TrainAccum acc{w, w + K, w + 2 * K, w + 3 * K, w + 3 * K + 1};
  const size_t acc_bytes = ((3 * (size_t)K + 2) * sizeof(unsigned long long) + 255) & ~(size_t)255;
  const int G = prefilter_grid_train(bits);
  void* table = G > 0 ? static_cast<char*>(d_ws) + acc_bytes : nullptr;
  const int nz = 3 * K + 2;
  k_zero_u64<<<(nz + 255) / 256, 256, 0, stream>>>(w, nz);
  k_init<<<(K + 255) / 256, 256, 0, stream>>>(samples, K, cb);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int threads = 512;
  const size_t smem = (size_t)K * (sizeof(float2) + 2 * sizeof(unsigned long long) + sizeof(unsigned));
  const void* fn = reinterpret_cast<const void*>(&k_assign);
  if ((err = allow_smem(fn, smem)) != cudaSuccess) return err;
  const int grid = persistent_grid(fn, threads, smem, (n + threads - 1) / threads);
  for (int it = 0; it < iters; ++it) {
    if (table != nullptr) {
      if ((err = launch_build_prefilter(d_codebook, bits, G, table, stream)) != cudaSuccess) return err;
    }
    k_assign<<<grid, threads, smem, stream>>>(samples, n, cb, K, table, acc, d_status);
    k_update<<<(K + 255) / 256, 256, 0, stream>>>(cb, K, acc, d_distortion, it);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace qamw
