// gemv.cu -- fused decode + skinny product y = x W_hat^T without forming W_hat.
//
// W_hat row i = r_i * diag(1/s) R_inv yhat_i with yhat_i pair k = sigma_k c[idx_ik]
// (paper section 3.2).  R_inv = R_fwd^T, so
//   y[t][i] = r_i * sum_k < xbar_t[k], c[idx_ik] >,  xbar_t = sigma (.) R_fwd(x_t / s)
// (pair k = coordinates 2k, 2k+1): the activation is rotated once and the
// weights are never decoded to BF16.
//
// batch 1 (k_gemv1): one persistent CTA per SM.  Each warp owns a fixed slice of
//   32 chunks (1024 pairs) and computes xbar for it straight into registers.
//   Tiles of R whole rows of packed indices stream into a 3-stage shared ring
//   through cp.async.bulk (TMA, mbarrier completion, bounded waits); codewords
//   come from an fp16x2 copy of the codebook replicated so that a warp's 32
//   random lookups hit at most 2 lanes per bank.  Per-slice partial dot
//   products are summed in a fixed order (bitwise reproducible).
// batch 2..16 (k_rotate + k_gemv_s): xbar for all columns is written once to
//   the workspace (chunk-interleaved so that lanes read consecutive words).
//   Each CTA stages 4 or 8 of its columns in shared memory beside a replicated
//   fp16x2 codebook, and a warp sums two rows at a time (batch 9..16: two
//   column passes).  Where that does not fit (long rows), k_gemv reads xbar
//   from the workspace with one warp per row.
#include <utility>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

// ------------------------------------------------------------------ batch 1

constexpr int kGemvStages = 3;

struct Gemv1Args {
  const uint8_t* packed;
  const __half* rnorm;
  const __half* sigma;
  const __half* scale;
  const __nv_bfloat16* x;
  const float2* codebook;
  __nv_bfloat16* y;
  int32_t* status;
  int64_t row_bytes;
  int d_out, d_in, block, K;
  uint64_t seed;
  int S;            // slices of 32 chunks per row
  int k;            // warps per slice
  int R;            // rows per tile (multiple of k)
  int ntiles;
  int copies_log2;  // codebook replicas (power of two)
  unsigned stage_bytes;
};

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

// acc += <xr pair q, fp16x2 codeword of index q> for the 32 indices packed in w
// (every index a compile-time constant, so xr stays in registers).
template <int BITS, int... Q>
__device__ __forceinline__ void dot_pairs(const uint32_t (&w)[BITS], const uint32_t* tab, int cl,
                                          uint32_t copy, const float (&xr)[kE], float& acc0,
                                          float& acc1, std::integer_sequence<int, Q...>) {
  (
      [&] {
        const uint32_t h = tab[(extract_idx<BITS, Q>(w) << cl) | copy];
        const float2 cw = __half22float2(*reinterpret_cast<const __half2*>(&h));
        acc0 = fmaf(xr[2 * Q], cw.x, acc0);
        acc1 = fmaf(xr[2 * Q + 1], cw.y, acc1);
      }(),
      ...);
}

// Region 0: the fp16x2 codebook table [K][copies], then xbar [64][C] (chunk-
// interleaved: D x / s first, then xbar in place).
__host__ __device__ inline size_t gemv1_table_bytes(int K, int copies_log2) {
  return align16((size_t)K * ((size_t)1 << copies_log2) * 4);
}
__host__ __device__ inline size_t gemv1_region0(int K, int copies_log2, int d_in) {
  return gemv1_table_bytes(K, copies_log2) + align16((size_t)d_in * 4);
}

__device__ __forceinline__ void issue_tile(const Gemv1Args& a, int tile, unsigned char* dst,
                                           uint64_t* bar) {
  const int r0 = tile * a.R, nr = min(a.R, a.d_out - r0);
  const unsigned bytes = (unsigned)(nr * a.row_bytes);
  mbar_expect_tx(bar, bytes);
  bulk_g2s(dst, a.packed + (int64_t)r0 * a.row_bytes, bytes, bar);
}

// Warps run through the tiles independently: after writing its partial dot
// products for a tile, each warp bumps the stage's counter; the warp that
// completes it sums the partials of every row of the tile (fixed order), writes
// y, and refills the stage with the tile kGemvStages ahead.
template <int BITS, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) k_gemv1(const Gemv1Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int copies = 1 << a.copies_log2;
  // region 0: first D x / s per column (d_in floats), then the fp16x2 codebook
  // table [K][copies]
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  unsigned char* stage = smem + gemv1_region0(a.K, a.copies_log2, a.d_in);
  float* partial = reinterpret_cast<float*>(stage + (size_t)kGemvStages * a.stage_bytes);
  const size_t part_floats = (size_t)a.R * a.S;
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(partial) +
                                              align16(kGemvStages * part_floats * 4));
  int* done = reinterpret_cast<int*>(bar + kGemvStages);
  int* issued = done + kGemvStages;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = a.d_in / kE;
  const int nwarps = a.S * a.k;

  if (tid == 0) {
    for (int s = 0; s < kGemvStages; ++s) {
      mbar_init(&bar[s], 1);
      done[s] = 0;
      issued[s] = 0;
    }
    fence_mbar_init();
  }
  // the fp16x2 codebook table needs nothing from the kernels ahead: `copies`
  // replicas of each entry side by side, written in a lane-rotated order,
  // (r + lane) mod copies, so that a warp's stores spread over the banks
#pragma unroll 4
  for (int j = tid; j < a.K; j += blockDim.x) {
    const float2 cw = __ldg(a.codebook + j);
    const __half2 h = __floats2half2_rn(cw.x, cw.y);
    const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
    for (int r = 0; r < copies; ++r)
      tab[(j << a.copies_log2) + ((r + lane) & (copies - 1))] = u;
  }
  // the indices, r_hat, sigma and s come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    // first tiles in flight while xbar is prepared
    for (int s = 0; s < kGemvStages; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile >= a.ntiles) break;
      issue_tile(a, tile, stage + (size_t)s * a.stage_bytes, &bar[s]);
      issued[s] = 1;
    }
  }
  // D_j x_j / s_j for every column into xsT [j][c] (8 columns per thread,
  // 16-byte loads); then one warp per slice turns its chunks into xbar =
  // sigma (.) R_fwd(x / s) in place, and every warp loads its chunk's xbar.
  float* xsT = reinterpret_cast<float*>(smem + gemv1_table_bytes(a.K, a.copies_log2));
  const uint64_t seed = a.seed;
  int flags = 0;
  for (int j8 = tid * 8; j8 < a.d_in; j8 += blockDim.x * 8) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.x + j8));
    const uint4 sv = __ldg(reinterpret_cast<const uint4*>(a.scale + j8));
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    const __half2* sh = reinterpret_cast<const __half2*>(&sv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 s2 = __half22float2(sh[e]);
      const float x0 = __uint_as_float(xw[e] << 16), x1 = __uint_as_float(xw[e] & 0xffff0000u);
      if (!isfinite(x0) || !isfinite(x1)) flags = QAMW_STATUS_NONFINITE;
      const int j = j8 + 2 * e;
      const float q0 = __fdiv_rn(x0, s2.x), q1 = __fdiv_rn(x1, s2.y);
      xsT[(j % kE) * C + j / kE] = mask_negative(seed, (uint32_t)j) ? -q0 : q0;
      xsT[((j + 1) % kE) * C + (j + 1) / kE] = mask_negative(seed, (uint32_t)(j + 1)) ? -q1 : q1;
    }
  }
  __syncthreads();

  const int sl = warp % a.S, kk = warp / a.S;
  const int c = sl * 32 + lane;
  const bool active = c < C;
  float xr[kE];
  if (kk == 0) {  // one warp per slice: xbar of its 32 chunks, in place
    if (active) {
#pragma unroll
      for (int j = 0; j < kE; ++j) xr[j] = xsT[j * C + c];
    } else {
#pragma unroll
      for (int j = 0; j < kE; ++j) xr[j] = 0.f;
    }
    fwht_reg<kE>(xr, min(a.block, kE));
    fwht_lanes<kE>(xr, max(a.block / kE, 1));
    if (active) {
      const float inv_sqrt_b = 1.0f / sqrtf((float)a.block);
      const uint4* sg8 = reinterpret_cast<const uint4*>(a.sigma + (int64_t)c * kQ);
#pragma unroll
      for (int t = 0; t < kQ / 8; ++t) {  // sigma of pairs 8t .. 8t + 7
        const uint4 v = __ldg(sg8 + t);
        const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f2 = __half22float2(h[e]);
          const int q = 8 * t + 2 * e;
          xsT[(2 * q) * C + c] = xr[2 * q] * (f2.x * inv_sqrt_b);
          xsT[(2 * q + 1) * C + c] = xr[2 * q + 1] * (f2.x * inv_sqrt_b);
          xsT[(2 * q + 2) * C + c] = xr[2 * q + 2] * (f2.y * inv_sqrt_b);
          xsT[(2 * q + 3) * C + c] = xr[2 * q + 3] * (f2.y * inv_sqrt_b);
        }
      }
    }
  }
  __syncthreads();
  if (active) {
#pragma unroll
    for (int j = 0; j < kE; ++j) xr[j] = xsT[j * C + c];
  } else {
#pragma unroll
    for (int j = 0; j < kE; ++j) xr[j] = 0.f;
  }

  const uint32_t copy = (uint32_t)lane & (uint32_t)(copies - 1);
  int it = 0;
  for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x, ++it) {
    const int st = it % kGemvStages;
    if (!mbar_wait_bounded(&bar[st], (unsigned)(it / kGemvStages) & 1u)) {
      flags |= QAMW_STATUS_TIMEOUT;
      break;
    }
    const int r0 = tile * a.R, nr = min(a.R, a.d_out - r0);
    const unsigned char* buf = stage + (size_t)st * a.stage_bytes;
    float* part = partial + st * part_floats;
    for (int rl = kk; rl < nr; rl += a.k) {
      float acc0 = 0.f, acc1 = 0.f;
      if (active) {
        const uint32_t* src =
            reinterpret_cast<const uint32_t*>(buf + (size_t)rl * a.row_bytes) + (size_t)c * BITS;
        uint32_t w[BITS];
#pragma unroll
        for (int t = 0; t < BITS; ++t) w[t] = src[t];
        dot_pairs<BITS>(w, tab, a.copies_log2, copy, xr, acc0, acc1,
                        std::make_integer_sequence<int, kQ>{});
      }
      float acc = acc0 + acc1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) part[rl * a.S + sl] = acc;
    }
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&done[st], 1) == nwarps - 1;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence_block();
      for (int r = lane; r < nr; r += 32) {
        float sum = 0.f;
        for (int s = 0; s < a.S; ++s) sum += part[r * a.S + s];
        a.y[r0 + r] = __float2bfloat16_rn(sum * __half2float(a.rnorm[r0 + r]));
      }
      __syncwarp();
      if (lane == 0) {
        done[st] = 0;
        const int next = tile + kGemvStages * gridDim.x;
        if (next < a.ntiles) {
          issue_tile(a, next, stage + (size_t)st * a.stage_bytes, &bar[st]);
          issued[st] += 1;
        }
      }
    }
  }
  // after a timeout: let the copies still in flight land before this CTA's
  // shared memory goes away
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < kGemvStages; ++s)
      if (issued[s] > 0) mbar_wait_bounded(&bar[s], (unsigned)(issued[s] - 1) & 1u);
  }
  raise_flag(a.status, flags);
}

// Shared memory of k_gemv1 for given replicas and tile rows.
size_t gemv1_smem(int K, int copies_log2, unsigned stage_bytes, int R, int S, int d_in) {
  return gemv1_region0(K, copies_log2, d_in) + (size_t)kGemvStages * stage_bytes +
         align16((size_t)kGemvStages * R * S * 4) + kGemvStages * sizeof(uint64_t) +
         2 * kGemvStages * sizeof(int);
}

template <int BITS>
cudaError_t run_gemv1(const qamw_matrix& m, const uint16_t* d_x, uint16_t* d_y,
                      int32_t* d_status, cudaStream_t stream) {
  Gemv1Args a;
  a.packed = m.packed;
  a.rnorm = reinterpret_cast<const __half*>(m.row_norm);
  a.sigma = reinterpret_cast<const __half*>(m.sigma);
  a.scale = reinterpret_cast<const __half*>(m.chan_scale);
  a.x = reinterpret_cast<const __nv_bfloat16*>(d_x);
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.y = reinterpret_cast<__nv_bfloat16*>(d_y);
  a.status = d_status;
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.d_in = m.d_in;
  a.block = m.block;
  a.K = 1 << m.bits;
  a.seed = m.mask_seed;
  const int C = m.d_in / kE;
  a.S = (C + 31) / 32;
  a.k = a.S <= 16 ? 16 / a.S : 1;  // 16 warps (512 threads) per SM
  // ~20 KB of indices per stage, whole rows, a multiple of k rows
  int R = (int)(20480 / m.row_bytes);
  R = R < a.k ? a.k : (R / a.k) * a.k;
  a.R = R;
  a.stage_bytes = (unsigned)(R * m.row_bytes);
  a.ntiles = (m.d_out + R - 1) / R;
  int cl = a.K <= 1024 ? 5 : 4;
  while (cl > 0 && gemv1_smem(a.K, cl, a.stage_bytes, R, a.S, a.d_in) > 227 * 1024) --cl;
  a.copies_log2 = cl;
  const size_t smem = gemv1_smem(a.K, cl, a.stage_bytes, R, a.S, a.d_in);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  const int threads = 32 * a.S * a.k;
  // 512 threads: at most 128 registers, 16 warps per SM
  const void* fn = threads <= 256 ? reinterpret_cast<const void*>(&k_gemv1<BITS, 256>)
                                  : reinterpret_cast<const void*>(&k_gemv1<BITS, 512>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = a.ntiles < sm_count() ? a.ntiles : sm_count();
  if (threads <= 256)
    return launch_pdl(k_gemv1<BITS, 256>, dim3(grid), dim3(threads), smem, stream, a);
  return launch_pdl(k_gemv1<BITS, 512>, dim3(grid), dim3(threads), smem, stream, a);
}

// ------------------------------------------------------------- batch 2..16

// xbarT[t][q][c] (float2) = pair 32c+q of xbar_t, for t < batch; zeros for
// batch <= t < bpad.  A CTA takes 32 consecutive (t, chunk c) items: all its
// threads form D x / s element by element into shared memory, then one warp
// rotates the 32 chunks from there (lane = item), so that the per-element
// divisions and sign hashes are spread over the whole CTA.
constexpr int kRotItems = 32;
constexpr int kRotThreads = 256;

__global__ void __launch_bounds__(kRotThreads) k_rotate(const __nv_bfloat16* __restrict__ x,
                                                        int batch, int bpad, int d_in, int block,
                                                        uint64_t seed,
                                                        const __half* __restrict__ s,
                                                        const __half* __restrict__ sigma,
                                                        float2* __restrict__ xbarT,
                                                        int32_t* status) {
  __shared__ float buf[kRotItems][kE + 1];  // +1: conflict-free rows and columns
  const int C = d_in / kE, P = d_in / 2;
  const int64_t V = (int64_t)bpad * C;
  const int nb = min(block, kE), lanes = max(block / kE, 1);
  const float inv_sqrt_b = 1.0f / sqrtf((float)block);
  int flags = 0;
  // s and sigma may come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  for (int64_t base = (int64_t)blockIdx.x * kRotItems; base < V;
       base += (int64_t)gridDim.x * kRotItems) {
    for (int e = threadIdx.x; e < kRotItems * kE; e += kRotThreads) {
      const int i = e / kE, j = e - i * kE;
      const int64_t v = base + i;
      const int64_t t = v < V ? v / C : bpad;
      float val = 0.f;
      if (t < batch) {
        const int col = (int)(v - t * C) * kE + j;
        const float xv = __bfloat162float(x[t * d_in + col]);
        if (!isfinite(xv)) flags = QAMW_STATUS_NONFINITE;
        const float q = __fdiv_rn(xv, __half2float(s[col]));
        val = mask_negative(seed, (uint32_t)col) ? -q : q;
      }
      buf[i][j] = val;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // one whole warp: the lane shuffles need all 32
      const int64_t v = base + threadIdx.x;
      const bool active = v < V;
      const int64_t t = active ? v / C : 0;
      const int c = active ? (int)(v - t * C) : 0;
      float xv[kE];
#pragma unroll
      for (int j = 0; j < kE; ++j) xv[j] = buf[threadIdx.x][j];
      fwht_reg<kE>(xv, nb);
      fwht_lanes<kE>(xv, lanes);
      if (active) {
        float sg[kQ];
        load_halves<kQ>(sigma + (int64_t)c * kQ, sg);
        float2* dst = xbarT + t * P + c;
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
          const float f = sg[q] * inv_sqrt_b;
          dst[(size_t)q * C] = make_float2(xv[2 * q] * f, xv[2 * q + 1] * f);
        }
      }
    }
    __syncthreads();
  }
  raise_flag(status, flags);
}

// One warp per output row; lanes take the row's 32-pair chunks round robin.
template <int BITS, int B>
__global__ void __launch_bounds__(256) k_gemv(const uint8_t* __restrict__ packed, int64_t row_bytes,
                                              const __half* __restrict__ rnorm,
                                              const float2* __restrict__ codebook, int K,
                                              const float2* __restrict__ xbarT, int d_out, int d_in,
                                              int batch, __nv_bfloat16* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char smem[];
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
      for (int q = 0; q < kQ; ++q) {
        const float2 cw = cb[idx[q]];
#pragma unroll
        for (int t = 0; t < B; ++t) {
          const float2 xb = __ldg(xbarT + (int64_t)t * P + (int64_t)q * C + c);
          acc[t] = fmaf(xb.x, cw.x, fmaf(xb.y, cw.y, acc[t]));
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

// The same product with B batch columns of xbar (columns t0 .. t0 + B - 1 of
// the workspace) staged in shared memory once per CTA.  A warp sums R
// consecutive rows at once, lanes over the rows' chunks, so that each xbar
// value read from shared memory serves R rows.  Codewords come from an fp16x2
// table with 2^cl replicas of each entry, lane l reading replica l mod 2^cl, as
// in the batch-1 kernel.  Used when B columns of xbar and the table fit in
// shared memory.
template <int BITS, int B, int R>
__global__ void __launch_bounds__(512, 1) k_gemv_s(const uint8_t* __restrict__ packed,
                                                   int64_t row_bytes, const __half* __restrict__ rnorm,
                                                   const float2* __restrict__ codebook, int K,
                                                   int cl, const float2* __restrict__ xbarT,
                                                   int t0, int d_out, int d_in, int batch,
                                                   __nv_bfloat16* __restrict__ y) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  float2* xs = reinterpret_cast<float2*>(smem + gemv1_table_bytes(K, cl));  // [B][P]
  const int C = d_in / kE, P = d_in / 2;
  const int lane = threadIdx.x & 31;
  const int copies = 1 << cl;
#pragma unroll 4
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const float2 cw = __ldg(codebook + j);
    const __half2 h = __floats2half2_rn(cw.x, cw.y);
    const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
    for (int r = 0; r < copies; ++r) tab[(j << cl) + ((r + lane) & (copies - 1))] = u;
  }
  const uint32_t copy = (uint32_t)lane & (uint32_t)(copies - 1);
  // xbar, the indices and r_hat come from the kernels ahead; the table build
  // above overlaps their end
  pdl_wait();
  pdl_trigger();
  {
    const float4* src = reinterpret_cast<const float4*>(xbarT + (int64_t)t0 * P);
    float4* dst = reinterpret_cast<float4*>(xs);
    const int n4 = B * P / 2;
#pragma unroll 4
    for (int i = threadIdx.x; i < n4; i += blockDim.x) dst[i] = __ldg(src + i);
  }
  __syncthreads();
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nt = min(B, batch - t0);
  for (int row = ((blockIdx.x * blockDim.x + threadIdx.x) >> 5) * R; row < d_out;
       row += warps * R) {
    float acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < B; ++t) acc[r][t] = 0.f;
    for (int c = lane; c < C; c += 32) {
      uint32_t idx[R][kQ];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        // rows past the end read index 0 and are not written
        uint32_t w[BITS];
        const bool ok = row + r < d_out;
        const uint32_t* src =
            reinterpret_cast<const uint32_t*>(packed + (int64_t)(ok ? row + r : row) * row_bytes);
#pragma unroll
        for (int t = 0; t < BITS; ++t) w[t] = ok ? __ldg(src + (size_t)c * BITS + t) : 0u;
        unpack32<BITS>(w, idx[r]);
      }
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        float2 cw[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t h = tab[(idx[r][q] << cl) | copy];
          cw[r] = __half22float2(*reinterpret_cast<const __half2*>(&h));
        }
#pragma unroll
        for (int t = 0; t < B; ++t) {
          const float2 xb = xs[t * P + q * C + c];
#pragma unroll
          for (int r = 0; r < R; ++r)
            acc[r][t] = fmaf(xb.x, cw[r].x, fmaf(xb.y, cw[r].y, acc[r][t]));
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < B; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], o);
      }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (row + r >= d_out) break;
        const float rn = __half2float(rnorm[row + r]);
#pragma unroll
        for (int t = 0; t < B; ++t)
          if (t < nt) y[(int64_t)(t0 + t) * d_out + row + r] = __float2bfloat16_rn(acc[r][t] * rn);
      }
    }
  }
}

constexpr size_t kGemvSmemCap = 200 * 1024;
constexpr int kGemvRows = 2;  // rows per warp in k_gemv_s

size_t gemv_s_smem(int K, int cl, int B, int d_in) {
  return gemv1_table_bytes(K, cl) + (size_t)B * (d_in / 2) * sizeof(float2);
}

// Most codebook replicas (up to 16, 32 for K <= 1024) with which the table and
// B columns of xbar fit in shared memory; -1 if not even one copy does.
int gemv_s_copies_log2(int K, int B, int d_in) {
  for (int cl = K <= 1024 ? 5 : 4; cl >= 0; --cl)
    if (gemv_s_smem(K, cl, B, d_in) <= kGemvSmemCap) return cl;
  return -1;
}

template <int BITS, int B, int R>
cudaError_t run_gemv_s(const qamw_matrix& m, int batch, int t0, int cl, const float2* xbar,
                       uint16_t* d_y, cudaStream_t stream) {
  const int threads = 512, K = 1 << m.bits;
  const size_t smem = gemv_s_smem(K, cl, B, m.d_in);
  const void* fn = reinterpret_cast<const void*>(&k_gemv_s<BITS, B, R>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int64_t warps = (m.d_out + R - 1) / R;
  const int grid = persistent_grid(fn, threads, smem, (warps * 32 + threads - 1) / threads);
  return launch_pdl(k_gemv_s<BITS, B, R>, dim3(grid), dim3(threads), smem, stream, m.packed,
                    m.row_bytes, reinterpret_cast<const __half*>(m.row_norm),
                    reinterpret_cast<const float2*>(m.codebook), K, cl,
                    static_cast<const float2*>(xbar), t0, m.d_out, m.d_in, batch,
                    reinterpret_cast<__nv_bfloat16*>(d_y));
}

template <int BITS>
cudaError_t gemv_bits(const qamw_matrix& m, const uint16_t* d_x, int batch, const float2* xbar,
                      uint16_t* d_y, int32_t* d_status, cudaStream_t stream) {
  if (batch == 1) return run_gemv1<BITS>(m, d_x, d_y, d_status, stream);
  const int K = 1 << m.bits;
  const int cl4 = gemv_s_copies_log2(K, 4, m.d_in), cl8 = gemv_s_copies_log2(K, 8, m.d_in);
  if (batch <= 4 && cl4 >= 0)
    return run_gemv_s<BITS, 4, kGemvRows>(m, batch, 0, cl4, xbar, d_y, stream);
  if (cl8 >= 0) {  // column passes of 8
    for (int t0 = 0; t0 < batch; t0 += 8) {
      const cudaError_t err =
          run_gemv_s<BITS, 8, kGemvRows>(m, batch, t0, cl8, xbar, d_y, stream);
      if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
  }
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
  if (batch > 1) {
    const int bpad = batch <= 4 ? 4 : (batch <= 8 ? 8 : 16);
    const int64_t V = (int64_t)bpad * (m.d_in / kE);
    const void* fn = reinterpret_cast<const void*>(&k_rotate);
    const int grid = persistent_grid(fn, kRotThreads, 0, (V + kRotItems - 1) / kRotItems);
    cudaError_t err = launch_pdl(k_rotate, dim3(grid), dim3(kRotThreads), 0, stream,
                                 reinterpret_cast<const __nv_bfloat16*>(d_x), batch, bpad,
                                 m.d_in, m.block, m.mask_seed,
                                 reinterpret_cast<const __half*>(m.chan_scale),
                                 reinterpret_cast<const __half*>(m.sigma), xbar, d_status);
    if (err != cudaSuccess) return err;
  }
  // The batch 2..16 kernels run B = 4/8/16 columns; columns batch..B-1 read
  // the zeroed xbar padding and are not written to y.
  switch (m.bits) {
    case 1: return gemv_bits<1>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 2: return gemv_bits<2>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 3: return gemv_bits<3>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 4: return gemv_bits<4>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 5: return gemv_bits<5>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 6: return gemv_bits<6>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 7: return gemv_bits<7>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 8: return gemv_bits<8>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 9: return gemv_bits<9>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 10: return gemv_bits<10>(m, d_x, batch, xbar, d_y, d_status, stream);
    case 11: return gemv_bits<11>(m, d_x, batch, xbar, d_y, d_status, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qamw
