// calibrate.cu -- the per-matrix side values of the QAM-W encoder, for one
// matrix or many in the same launches:
//   k_scales        s_j = binary16((a_j / mean a)^alpha)   (activation-aware
//                   per-channel scaling; one CTA per matrix)
//   k_calib_rows    |z_k| sums over the first 1024 rows    (paper section 3.4,
//                   eq. 1; 32 CTAs of 32 rows per matrix)
//   k_calib_ext     later rows when those held zero rows   (one CTA per matrix)
//   k_calib_finish  sigma_k = binary16(sum / (n sqrt(pi/2)))
// A launch covers up to kCalMany matrices (their shapes may differ); a list of
// 224 matrices takes four launches per 64 instead of four per matrix.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

struct CalibMat {
  const void* W;       // [d_out][d_in], T
  const float* act;    // [d_in] activation statistic, nullable (s = 1)
  __half* s;           // [d_in] channel scales (written by k_scales)
  __half* sigma;       // [d_in / 2]
  float* partial;      // [kCalCtas][d_in / 2] |z_k| sums of each CTA's rows
  float* ext;          // [d_in / 2] sums of the rows past 1023
  int32_t* nonzero;    // [kCalCtas] non-zero rows each CTA found
  int32_t* n_cal;      // [1] rows eq. (1) averages over
  int d_out, d_in, block;
  uint64_t seed;
};

template <int MAXM>
struct CalibLaunch {
  CalibMat m[MAXM];
  int n;
  float alpha;
  int32_t* status;
};

constexpr int kCalMany = 64;

// ------------------------------------------------------------------ scales

// One CTA of 1024 threads per matrix: thread t holds the statistic of channels
// t + 1024 i (i < 32, d_in <= 32768) in registers, so the statistic is read
// once; the fp64 sum is reduced in a fixed order (per-thread ascending i, a
// shuffle tree per warp, then the 32 warp sums by the same tree), so the mean
// is bitwise reproducible; each thread then rounds its own channels' scales.
// Without a statistic (or with alpha = 0) every scale is 1.
constexpr int kScaleThreads = 1024;
template <int MAXM>
__global__ void __launch_bounds__(kScaleThreads) k_scales(const __grid_constant__ CalibLaunch<MAXM> L) {
  __shared__ double red[32];
  __shared__ double mean_s;
  const CalibMat& M = L.m[blockIdx.x];
  const int d_in = M.d_in;
  const float alpha = L.alpha;
  if (M.act == nullptr || alpha == 0.0f) {
    pdl_wait();  // s may still be read by the kernel ahead
    pdl_trigger();
    for (int j = threadIdx.x; j < d_in; j += kScaleThreads) M.s[j] = __float2half(1.0f);
    return;
  }
  constexpr int kPer = kMaxDin / kScaleThreads;
  float vals[kPer];
  double sum = 0.0;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = threadIdx.x + i * kScaleThreads;
    vals[i] = j < d_in ? M.act[j] : 1.f;
    if (j < d_in) {
      if (vals[i] > 0.f && isfinite(vals[i]))
        sum += (double)vals[i];
      else
        bad = 1;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    double t = red[threadIdx.x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) mean_s = t / (double)d_in;
  }
  bad = __syncthreads_or(bad);
  const double mean = mean_s;
  pdl_wait();  // s may still be read by the kernel ahead
  pdl_trigger();
  int range = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = threadIdx.x + i * kScaleThreads;
    if (j >= d_in) break;
    const float v = vals[i];
    __half h;
    if (v > 0.f && isfinite(v)) {
      // binary16(pow(v / mean, alpha)) of the fp64 power: an fp32 evaluation
      // decides unless it lies within its error bound (log2f 1 ulp, exp2f 2
      // ulp, the ratio 2^-24: under (2 + |t| + |alpha|) 2^-23 relative for
      // t = alpha log2 r; a 2x margin taken) of a binary16 rounding midpoint -- the
      // midpoints between h and its neighbours are exact in fp32 -- or
      // outside the normal/subnormal range; there the fp64 pow decides
      const float t = alpha * log2f((float)((double)v / mean));
      const float y = exp2f(t);
      h = __float2half_rn(y);
      const uint16_t hb = __half_as_ushort(h);
      bool exact = y > 0.f && hb > 0u && hb < 0x7bffu;
      if (exact) {
        const float hf = __half2float(h);
        const float up = __half2float(__ushort_as_half((uint16_t)(hb + 1)));
        const float dn = __half2float(__ushort_as_half((uint16_t)(hb - 1)));
        const float tol = y * (2.0f + fabsf(t) + fabsf(alpha)) * 2.4e-7f;
        exact = fabsf(y - 0.5f * (hf + up)) > tol && fabsf(y - 0.5f * (hf + dn)) > tol;
      }
      if (!exact) h = __double2half(pow((double)v / mean, (double)alpha));
      const float hf2 = __half2float(h);
      if (isinf(hf2) || hf2 == 0.f) range = 1;
    } else {
      h = __float2half(1.0f);
    }
    M.s[j] = h;
  }
  raise_flag(L.status, ((threadIdx.x == 0 && bad) ? QAMW_STATUS_BAD_STAT : 0) |
                           (range ? QAMW_STATUS_RANGE : 0));
}

// ------------------------------------------------------------- calibration

// Eq. (1) over the first min(1024, #non-zero) non-zero rows:
//   k_calib_rows   CTA (b, i) takes rows [32b, 32b + 32) of matrix i's first
//                  1024: row norm (fixed-order reduction), rotation, |z_k| / r
//                  summed over its non-zero rows into partial[b][k];
//                  nonzero[b] = their count.  RPC = min(32, 512 / C) rows at a
//                  time, thread (g, c) holding chunk c of row g of the batch.
//   k_calib_ext    if the first 1024 rows held zero rows, one CTA walks on
//                  from row 1024 in order, adding the next non-zero rows into
//                  ext[k] until there are 1024 (a path only matrices with zero
//                  rows take); else it only records the count.
//   k_calib_finish sigma_k = binary16((sum_b partial[b][k] + ext[k]) /
//                  (n sqrt(pi/2))), 1 when that rounds to 0.
constexpr int kCalThreads = 512;
constexpr int kCalPer = kCalRows / kCalCtas;  // rows per CTA: 32
// k_calib_rows gives each thread CE consecutive columns of a row: 32 (16 pairs)
// when every matrix of the launch has d_in <= 32 x 512, so that a thread's
// values and sums fit its registers with two CTAs per SM, else 64.  The
// butterflies give bitwise the same rotation for either width.
constexpr int kCalNarrow = 32;
constexpr int kCalNarrowMaxDin = kCalNarrow * kCalThreads;

__host__ __device__ inline int calib_rpc(int d_in, int ce) {
  const int r = kCalThreads / (d_in / ce);
  return r < 1 ? 1 : (r > kCalPer ? kCalPer : r);
}

// Shared memory of k_calib_rows for a matrix: fT4 [d_in / 4] (quads of a
// CE-column chunk) | red [RPC][P] | part [512] | rsum [32].
__host__ __device__ inline size_t calib_rows_smem(int d_in, int ce) {
  return ((size_t)d_in + (size_t)calib_rpc(d_in, ce) * (d_in / 2) + kCalThreads + kCalPer) *
         sizeof(float);
}

// N consecutive values of a row as fp32.
template <int N>
__device__ __forceinline__ void load_cols(const float* p, float (&x)[N]) {
  const float4* s4 = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int t = 0; t < N / 4; ++t) {
    const float4 v = __ldg(s4 + t);
    x[4 * t] = v.x;
    x[4 * t + 1] = v.y;
    x[4 * t + 2] = v.z;
    x[4 * t + 3] = v.w;
  }
}
template <int N>
__device__ __forceinline__ void load_cols(const __nv_bfloat16* p, float (&x)[N]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int t = 0; t < N / 8; ++t) {
    const uint4 v = __ldg(s4 + t);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * t + 2 * e] = __uint_as_float(u[e] << 16);
      x[8 * t + 2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
    }
  }
}

template <typename T, int MAXM, int kCE>
__global__ void __launch_bounds__(kCalThreads, kCE == kCalNarrow ? 2 : 1)
    k_calib_rows(const __grid_constant__ CalibLaunch<MAXM> L) {
  extern __shared__ __align__(16) float sm[];
  constexpr int kQh = kCE / 2;  // pairs per thread
  const CalibMat& M = L.m[blockIdx.y];
  const T* __restrict__ W = static_cast<const T*>(M.W);
  const int d_in = M.d_in, C = d_in / kCE, P = d_in / 2;
  const int RPC = calib_rpc(d_in, kCE);
  float4* fT4 = reinterpret_cast<float4*>(sm);  // [j/4][c]: D * s of columns kCE c + j .. + 3
  float* red = sm + d_in;               // [g][q][c]
  float* part = red + (size_t)RPC * P;  // [blockDim] partial sums of squares
  float* rsum = part + kCalThreads;     // [RPC]
  pdl_wait();  // s comes from the kernel ahead
  pdl_trigger();
  const uint64_t seed = M.seed;
  fill_quads<kCE>(fT4, M.s, d_in, C, [=](int j, float v) {
    return mask_negative(seed, (uint32_t)j) ? -v : v;
  });
  __syncthreads();
  const int g = threadIdx.x / C, c = threadIdx.x - g * C;
  const bool lane_ok = g < RPC;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = kCalThreads >> 5;
  const int nb = min(M.block, kCE), lanes = max(M.block / kCE, 1);
  const float inv_sqrt_b = 1.0f / sqrtf((float)M.block);
  const int rows = min(M.d_out, kCalRows);
  const int t0 = blockIdx.x * kCalPer, t1 = min(t0 + kCalPer, rows);
  float acc[kQh];
#pragma unroll
  for (int q = 0; q < kQh; ++q) acc[q] = 0.f;
  int nz = 0, flags = 0;
  for (int base = t0; base < t1; base += RPC) {
    const int row = base + g;
    const bool active = lane_ok && row < t1;
    float x[kCE];
    float ss = 0.f;
    if (active) {
      load_cols<kCE>(W + (int64_t)row * d_in + (int64_t)c * kCE, x);
#pragma unroll
      for (int i = 0; i < kCE / 4; ++i) {  // four factors per 16-byte load, element order kept
        const float4 f = fT4[i * C + c];
        x[4 * i] *= f.x;
        ss = fmaf(x[4 * i], x[4 * i], ss);
        x[4 * i + 1] *= f.y;
        ss = fmaf(x[4 * i + 1], x[4 * i + 1], ss);
        x[4 * i + 2] *= f.z;
        ss = fmaf(x[4 * i + 2], x[4 * i + 2], ss);
        x[4 * i + 3] *= f.w;
        ss = fmaf(x[4 * i + 3], x[4 * i + 3], ss);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kCE; ++j) x[j] = 0.f;
    }
    part[threadIdx.x] = ss;
    fwht_reg<kCE>(x, nb);
    fwht_lanes<kCE>(x, lanes);
    __syncthreads();
    for (int q = warp; q < RPC; q += nwarps) {
      float t = 0.f;
      for (int k = lane; k < C; k += 32) t += part[q * C + k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) rsum[q] = sqrtf(t);
    }
    __syncthreads();
    if (active) {
      const float r = rsum[g];
      if (!isfinite(r)) flags = QAMW_STATUS_NONFINITE;
      if (r > 0.f) {
        if (c == 0) ++nz;
        const float inv = inv_sqrt_b / r;
#pragma unroll
        for (int q = 0; q < kQh; ++q) {
          const float zx = x[2 * q] * inv, zy = x[2 * q + 1] * inv;
          acc[q] += sqrtf(fmaf(zx, zx, zy * zy));
        }
      }
    }
    __syncthreads();  // part / rsum are rewritten by the next batch
  }
  if (lane_ok) {
#pragma unroll
    for (int q = 0; q < kQh; ++q) red[(size_t)g * P + q * C + c] = acc[q];
  }
  // non-zero rows of this CTA: thread (g, 0) counted those of group g
  __shared__ int cnt_sh;
  if (threadIdx.x == 0) cnt_sh = 0;
  __syncthreads();
  if (nz) atomicAdd(&cnt_sh, nz);
  for (int k = threadIdx.x; k < P; k += kCalThreads) {
    float v = 0.f;
    for (int gg = 0; gg < RPC; ++gg) v += red[(size_t)gg * P + (k % kQh) * C + k / kQh];
    M.partial[(size_t)blockIdx.x * P + k] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) M.nonzero[blockIdx.x] = cnt_sh;
  raise_flag(L.status, flags);
}

// One CTA per matrix of kCalThreads >= C threads; thread c < C holds chunk c of
// the current row.
template <typename T, int MAXM>
__global__ void __launch_bounds__(kCalThreads) k_calib_ext(const __grid_constant__ CalibLaunch<MAXM> L) {
  extern __shared__ __align__(16) float4 fT4[];  // [j/4][c]
  __shared__ float part[kCalThreads];
  __shared__ float rtot;
  __shared__ int total;
  const CalibMat& M = L.m[blockIdx.x];
  const T* __restrict__ W = static_cast<const T*>(M.W);
  const int d_in = M.d_in, d_out = M.d_out, C = d_in / kE;
  pdl_wait();
  pdl_trigger();
  const int c = threadIdx.x;
  const bool active_c = c < C;
  if (threadIdx.x < 32) {  // the non-zero rows found among the first 1024 (integer sum)
    int n = 0;
    for (int b = threadIdx.x; b < kCalCtas; b += 32) n += M.nonzero[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if (threadIdx.x == 0) total = n;
  }
  float acc[kQ];
#pragma unroll
  for (int q = 0; q < kQ; ++q) acc[q] = 0.f;
  __syncthreads();
  if (total < kCalRows && d_out > kCalRows) {
    const uint64_t seed = M.seed;
    fill_quads<kE>(fT4, M.s, d_in, C, [=](int j, float v) {
      return mask_negative(seed, (uint32_t)j) ? -v : v;
    });
    __syncthreads();
    const int nb = min(M.block, kE), lanes = max(M.block / kE, 1);
    const float inv_sqrt_b = 1.0f / sqrtf((float)M.block);
    for (int row = kCalRows; row < d_out && total < kCalRows; ++row) {
      float x[kE];
      float ss = 0.f;
      if (active_c) {
        load64(W + (int64_t)row * d_in + (int64_t)c * kE, x);
#pragma unroll
        for (int i = 0; i < kE / 4; ++i) {
          const float4 f = fT4[i * C + c];
          x[4 * i] *= f.x;
          ss = fmaf(x[4 * i], x[4 * i], ss);
          x[4 * i + 1] *= f.y;
          ss = fmaf(x[4 * i + 1], x[4 * i + 1], ss);
          x[4 * i + 2] *= f.z;
          ss = fmaf(x[4 * i + 2], x[4 * i + 2], ss);
          x[4 * i + 3] *= f.w;
          ss = fmaf(x[4 * i + 3], x[4 * i + 3], ss);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kE; ++j) x[j] = 0.f;
      }
      part[threadIdx.x] = ss;
      fwht_reg<kE>(x, nb);
      fwht_lanes<kE>(x, lanes);
      __syncthreads();
      if (threadIdx.x < 32) {
        float t = 0.f;
        for (int k = threadIdx.x; k < C; k += 32) t += part[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) rtot = sqrtf(t);
      }
      __syncthreads();
      const float r = rtot;
      if (r > 0.f && active_c) {
        const float inv = inv_sqrt_b / r;
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
          const float zx = x[2 * q] * inv, zy = x[2 * q + 1] * inv;
          acc[q] += sqrtf(fmaf(zx, zx, zy * zy));
        }
      }
      __syncthreads();
      if (threadIdx.x == 0 && r > 0.f) ++total;
      __syncthreads();
    }
  }
  if (active_c) {
#pragma unroll
    for (int q = 0; q < kQ; ++q) M.ext[c * kQ + q] = acc[q];
  }
  if (threadIdx.x == 0) *M.n_cal = min(total, kCalRows);
}

// 16 threads per pair k: thread i sums partials i, i+16, ... in fp64, then the
// 16 sums are combined by a fixed shuffle tree (deterministic).  blockIdx.y is
// the matrix.
template <int MAXM>
__global__ void __launch_bounds__(256) k_calib_finish(const __grid_constant__ CalibLaunch<MAXM> L) {
  pdl_wait();
  pdl_trigger();
  const CalibMat& M = L.m[blockIdx.y];
  const int P = M.d_in / 2;
  const int g = blockIdx.x * 16 + threadIdx.x / 16, i = threadIdx.x & 15;
  if (blockIdx.x * 16 >= P) return;  // the whole CTA: past this matrix's pairs
  const int k = min(g, P - 1);
  double sum = 0.0;
#pragma unroll 2
  for (int p = i; p < kCalCtas; p += 16) sum += (double)M.partial[(size_t)p * P + k];
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (i != 0 || g >= P) return;
  sum += (double)M.ext[k];
  const int n = *M.n_cal;
  const double rayleigh = 1.2533141373155002512;  // sqrt(pi/2)
  __half h = __double2half(n > 0 ? sum / (double)n / rayleigh : 0.0);
  const float hf = __half2float(h);
  if (hf == 0.f) h = __float2half(1.0f);
  if (isinf(hf)) raise_flag(L.status, QAMW_STATUS_RANGE);
  M.sigma[k] = h;
}

template <typename T, int MAXM>
cudaError_t calibrate_group(const CalibLaunch<MAXM>& L, bool scales, bool sigma, cudaStream_t stream) {
  cudaError_t err;
  if (scales) {
    err = launch_pdl(k_scales<MAXM>, dim3(L.n), dim3(kScaleThreads), 0, stream, L);
    if (err != cudaSuccess) return err;
  }
  if (!sigma) return cudaSuccess;
  size_t esmem = 0;
  int pmax = 0, dmax = 0;
  for (int i = 0; i < L.n; ++i) {
    esmem = std::max(esmem, (size_t)L.m[i].d_in * sizeof(float));
    pmax = std::max(pmax, L.m[i].d_in / 2);
    dmax = std::max(dmax, L.m[i].d_in);
  }
  const int ce = dmax <= kCalNarrowMaxDin ? kCalNarrow : kE;
  size_t smem = 0;
  for (int i = 0; i < L.n; ++i) smem = std::max(smem, calib_rows_smem(L.m[i].d_in, ce));
  const void* fn = ce == kCalNarrow ? reinterpret_cast<const void*>(&k_calib_rows<T, MAXM, kCalNarrow>)
                                    : reinterpret_cast<const void*>(&k_calib_rows<T, MAXM, kE>);
  if ((err = allow_smem(fn, smem)) != cudaSuccess) return err;
  if (ce == kCalNarrow)
    err = launch_pdl(k_calib_rows<T, MAXM, kCalNarrow>, dim3(kCalCtas, L.n), dim3(kCalThreads), smem,
                     stream, L);
  else
    err = launch_pdl(k_calib_rows<T, MAXM, kE>, dim3(kCalCtas, L.n), dim3(kCalThreads), smem, stream,
                     L);
  if (err != cudaSuccess) return err;
  const void* efn = reinterpret_cast<const void*>(&k_calib_ext<T, MAXM>);
  if ((err = allow_smem(efn, esmem)) != cudaSuccess) return err;
  err = launch_pdl(k_calib_ext<T, MAXM>, dim3(L.n), dim3(kCalThreads), esmem, stream, L);
  if (err != cudaSuccess) return err;
  return launch_pdl(k_calib_finish<MAXM>, dim3((pmax + 15) / 16, L.n), dim3(256), 0, stream, L);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of one matrix: nonzero [32] | n_cal | ext [P] | partial [32][P].
size_t calib_ws_one(int d_in, CalibMat* carve, char* base) {
  const size_t P = (size_t)d_in / 2;
  size_t off = 0;
  const size_t o_nz = off;
  off += align256(kCalCtas * sizeof(int32_t));
  const size_t o_n = off;
  off += align256(sizeof(int32_t));
  const size_t o_ext = off;
  off += align256(P * sizeof(float));
  const size_t o_part = off;
  off += align256((size_t)kCalCtas * P * sizeof(float));
  if (carve) {
    carve->nonzero = reinterpret_cast<int32_t*>(base + o_nz);
    carve->n_cal = reinterpret_cast<int32_t*>(base + o_n);
    carve->ext = reinterpret_cast<float*>(base + o_ext);
    carve->partial = reinterpret_cast<float*>(base + o_part);
  }
  return off;
}

template <int MAXM>
void describe(CalibLaunch<MAXM>& L, int i, const void* W, const float* act, const qamw_matrix& m,
              char* ws) {
  CalibMat& c = L.m[i];
  c.W = W;
  c.act = act;
  c.s = reinterpret_cast<__half*>(m.chan_scale);
  c.sigma = reinterpret_cast<__half*>(m.sigma);
  c.d_out = m.d_out;
  c.d_in = m.d_in;
  c.block = m.block;
  c.seed = m.mask_seed;
  calib_ws_one(m.d_in, &c, ws);
}

template <typename T>
cudaError_t calibrate_many_typed(const void* const* W, const float* const* act, float alpha,
                                 const qamw_matrix* ms, int n, bool scales, bool sigma, char* ws,
                                 int32_t* st, cudaStream_t stream) {
  // one group of up to kCalMany matrices at a time, each with its own part of
  // the workspace; a one-matrix call goes through the same kernels
  if (n == 1) {
    CalibLaunch<1> L;
    L.n = 1;
    L.alpha = alpha;
    L.status = st;
    describe(L, 0, W ? W[0] : nullptr, act ? act[0] : nullptr, ms[0], ws);
    return calibrate_group<T, 1>(L, scales, sigma, stream);
  }
  size_t off = 0;
  for (int i0 = 0; i0 < n; i0 += kCalMany) {
    CalibLaunch<kCalMany> L;
    L.n = std::min(kCalMany, n - i0);
    L.alpha = alpha;
    L.status = st;
    for (int i = 0; i < L.n; ++i) {
      const qamw_matrix& m = ms[i0 + i];
      describe(L, i, W ? W[i0 + i] : nullptr, act ? act[i0 + i] : nullptr, m, ws + off);
      off += calib_ws_one(m.d_in, nullptr, nullptr);
    }
    const cudaError_t err = calibrate_group<T, kCalMany>(L, scales, sigma, stream);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

size_t calibrate_workspace_bytes(int d_out, int d_in, EncodeWorkspace* carve, void* base) {
  (void)d_out;
  CalibMat c;
  const size_t bytes = calib_ws_one(d_in, carve ? &c : nullptr, static_cast<char*>(base));
  if (carve) {
    carve->cal_nonzero = c.nonzero;
    carve->n_cal = c.n_cal;
    carve->cal_ext = c.ext;
    carve->cal_partial = c.partial;
    carve->prefilter = nullptr;
  }
  return bytes;
}

size_t calibrate_many_workspace_bytes(const qamw_matrix* ms, int n) {
  size_t b = 0;
  for (int i = 0; i < n; ++i) b += calib_ws_one(ms[i].d_in, nullptr, nullptr);
  return b;
}

cudaError_t launch_channel_scales(const float* d_act_stat, int d_in, float alpha, uint16_t* d_scale,
                                  int32_t* d_status, cudaStream_t stream) {
  qamw_matrix m{};
  m.d_in = d_in;
  m.block = 1;
  m.chan_scale = d_scale;
  const float* act[1] = {d_act_stat};
  return calibrate_many_typed<float>(nullptr, act, alpha, &m, 1, true, false, nullptr, d_status,
                                     stream);
}

cudaError_t launch_calibrate(const void* d_W, int dtype, const qamw_matrix& m,
                             const EncodeWorkspace& ws, int32_t* d_status, cudaStream_t stream) {
  // the workspace carve of calibrate_workspace_bytes starts at cal_nonzero
  char* base = reinterpret_cast<char*>(ws.cal_nonzero);
  const void* W[1] = {d_W};
  if (dtype == QAMW_DTYPE_F32)
    return calibrate_many_typed<float>(W, nullptr, 0.f, &m, 1, false, true, base, d_status, stream);
  return calibrate_many_typed<__nv_bfloat16>(W, nullptr, 0.f, &m, 1, false, true, base, d_status,
                                             stream);
}

cudaError_t launch_calibrate_many(const void* const* d_W, int dtype, const float* const* d_act,
                                  float alpha, const qamw_matrix* ms, int n, void* d_ws,
                                  int32_t* d_status, cudaStream_t stream) {
  char* base = static_cast<char*>(d_ws);
  if (dtype == QAMW_DTYPE_F32)
    return calibrate_many_typed<float>(d_W, d_act, alpha, ms, n, true, true, base, d_status, stream);
  return calibrate_many_typed<__nv_bfloat16>(d_W, d_act, alpha, ms, n, true, true, base, d_status,
                                             stream);
}

}  // namespace qamw
