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
//   Tiles of R whole rows of packed indices (~45 KB) stream into a 2-stage shared ring
//   through cp.async.bulk (TMA, mbarrier completion, bounded waits); codewords
//   come from an fp16x2 copy of the codebook replicated so that a warp's 32
//   random lookups hit at most 2 lanes per bank.  Per-slice partial dot
//   products are summed in a fixed order (bitwise reproducible).
// batch 2..16 (k_rotate_mma + k_gemv_mma): x_bar for 8 or 16 columns is
//   written once to the workspace in the operand order of the tensor cores;
//   16-row tiles are products of gathered codewords with x_bar on m16n8k16
//   MMAs (binary16 high/low parts, fp32 accumulation), the packed indices
//   streaming into shared memory through per-warp bulk-copy rings.
#include <utility>
#include <vector>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

// ------------------------------------------------------------------ batch 1

constexpr int kGemvStages = 2;
// Index bytes per tile of whole rows: two or more rows per warp at the common
// widths, so a warp's per-tile cost (its wait, its share of the row sums)
// spreads over more pairs.
constexpr int kGemvTileBytes = 46080;

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
  // ~45 KB of indices per stage, whole rows, a multiple of k rows
  int R = (int)(kGemvTileBytes / m.row_bytes);
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

// ------------------------------------------------ batch 1, many matrices
//
// qamw_decode_gemv_many: x_bar of every matrix is formed once, by
// k_xbar1_many, into the workspace as [chunk][64] floats -- the arithmetic of
// k_gemv1's own preparation, so the products are bitwise those of single calls
// -- and one persistent launch per run of matrices with the same d_in, block,
// bits and codebook (k_gemv1_many) builds the replicated codebook table once
// and streams the tiles of all of them.  Each CTA takes a contiguous range of
// the run's (matrix, tile) sequence and reloads its lanes' x_bar only where the
// matrix changes.

constexpr int kGemvManyMax = 64;
constexpr int kGemvManyStages = kGemvStages;       // ring depth of k_gemv1_many
constexpr int kGemvManyTileBytes = kGemvTileBytes;  // index bytes per tile (whole rows)
constexpr int kXb1Threads = 128;

struct Xbar1Mat {
  const __nv_bfloat16* x;
  const __half* sigma;
  const __half* scale;
  float* xbar;  // [C][64]
  uint64_t seed;
};

template <int MAXM>
struct Xbar1Args {
  Xbar1Mat m[MAXM];
  int32_t* status;
  int n, d_in, block;
};

// One lane per (matrix, chunk), matrices consecutive, chunks of a matrix in
// consecutive lanes (a block > 64 spans lanes of one matrix: C is a multiple of
// block / 64).
template <int MAXM>
__global__ void __launch_bounds__(kXb1Threads) k_xbar1_many(const __grid_constant__ Xbar1Args<MAXM> a) {
  const int C = a.d_in / kE;
  const int64_t V = (int64_t)a.n * C;
  const int64_t v = (int64_t)blockIdx.x * kXb1Threads + threadIdx.x;
  const bool active = v < V;
  const int mi = active ? (int)(v / C) : 0;
  const int c = active ? (int)(v - (int64_t)mi * C) : 0;
  const Xbar1Mat& M = a.m[mi];
  int flags = 0;
  pdl_wait();
  pdl_trigger();
  float xr[kE];
  if (active) {
    const uint4* xp = reinterpret_cast<const uint4*>(M.x + (int64_t)c * kE);
    const uint4* sp = reinterpret_cast<const uint4*>(M.scale + (int64_t)c * kE);
#pragma unroll
    for (int t = 0; t < kE / 8; ++t) {
      const uint4 xv = __ldg(xp + t);
      const uint4 sv = __ldg(sp + t);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
      const __half2* sh = reinterpret_cast<const __half2*>(&sv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 s2 = __half22float2(sh[e]);
        const float x0 = __uint_as_float(xw[e] << 16), x1 = __uint_as_float(xw[e] & 0xffff0000u);
        if (!isfinite(x0) || !isfinite(x1)) flags = QAMW_STATUS_NONFINITE;
        const int j = 8 * t + 2 * e, col = c * kE + j;
        const float q0 = __fdiv_rn(x0, s2.x), q1 = __fdiv_rn(x1, s2.y);
        xr[j] = mask_negative(M.seed, (uint32_t)col) ? -q0 : q0;
        xr[j + 1] = mask_negative(M.seed, (uint32_t)(col + 1)) ? -q1 : q1;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < kE; ++j) xr[j] = 0.f;
  }
  fwht_reg<kE>(xr, min(a.block, kE));
  fwht_lanes<kE>(xr, max(a.block / kE, 1));
  if (active) {
    const float inv_sqrt_b = 1.0f / sqrtf((float)a.block);
    const uint4* sg8 = reinterpret_cast<const uint4*>(M.sigma + (int64_t)c * kQ);
    float4* dst = reinterpret_cast<float4*>(M.xbar + (int64_t)c * kE);
#pragma unroll
    for (int t = 0; t < kQ / 8; ++t) {  // sigma of pairs 8t .. 8t + 7
      const uint4 u = __ldg(sg8 + t);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f2 = __half22float2(h[e]);
        const int q = 8 * t + 2 * e;
        dst[q / 2] = make_float4(xr[2 * q] * (f2.x * inv_sqrt_b), xr[2 * q + 1] * (f2.x * inv_sqrt_b),
                                 xr[2 * q + 2] * (f2.y * inv_sqrt_b),
                                 xr[2 * q + 3] * (f2.y * inv_sqrt_b));
      }
    }
  }
  raise_flag(a.status, flags);
}

struct Gemv1ManyMat {
  const uint8_t* packed;
  const __half* rnorm;
  const float* xbar;  // [C][64]
  __nv_bfloat16* y;
  int64_t tile0;  // first tile of this matrix in the run
  int d_out;
};

template <int MAXM>
struct Gemv1ManyArgs {
  Gemv1ManyMat m[MAXM];
  const float2* codebook;
  int32_t* status;
  int64_t row_bytes;
  int64_t ntiles;
  int n, d_in, K, S, k, R, copies_log2;
  unsigned stage_bytes;
};

// Shared memory of k_gemv1_many: the table, the ring, the partial sums, bars.
size_t gemv1_many_smem(int K, int copies_log2, unsigned stage_bytes, int R, int S) {
  return gemv1_table_bytes(K, copies_log2) + (size_t)kGemvManyStages * stage_bytes +
         align16((size_t)kGemvManyStages * R * S * 4) + kGemvManyStages * sizeof(uint64_t) +
         2 * kGemvManyStages * sizeof(int);
}

template <int BITS, int MAXT, int MAXM>
__global__ void __launch_bounds__(MAXT, 1) k_gemv1_many(const __grid_constant__ Gemv1ManyArgs<MAXM> a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int copies = 1 << a.copies_log2;
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  unsigned char* stage = smem + gemv1_table_bytes(a.K, a.copies_log2);
  float* partial = reinterpret_cast<float*>(stage + (size_t)kGemvManyStages * a.stage_bytes);
  const size_t part_floats = (size_t)a.R * a.S;
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(partial) +
                                              align16(kGemvManyStages * part_floats * 4));
  int* done = reinterpret_cast<int*>(bar + kGemvManyStages);
  int* issued = done + kGemvManyStages;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = a.d_in / kE;
  const int nwarps = a.S * a.k;

  if (tid == 0) {
    for (int s = 0; s < kGemvManyStages; ++s) {
      mbar_init(&bar[s], 1);
      done[s] = 0;
      issued[s] = 0;
    }
    fence_mbar_init();
  }
  // the fp16x2 codebook table (as k_gemv1's) needs nothing from the kernels ahead
#pragma unroll 4
  for (int j = tid; j < a.K; j += blockDim.x) {
    const float2 cw = __ldg(a.codebook + j);
    const __half2 h = __floats2half2_rn(cw.x, cw.y);
    const uint32_t u = *reinterpret_cast<const uint32_t*>(&h);
    for (int r = 0; r < copies; ++r)
      tab[(j << a.copies_log2) + ((r + lane) & (copies - 1))] = u;
  }
  __syncthreads();
  // the indices, r_hat and x_bar come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  const int64_t t_lo = (int64_t)blockIdx.x * a.ntiles / gridDim.x;
  const int64_t t_hi = ((int64_t)blockIdx.x + 1) * a.ntiles / gridDim.x;
  // the matrix whose tiles hold tile t (tile0 ascending)
  auto mat_of = [&](int64_t t) {
    int lo = 0, hi = a.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.m[mid].tile0 <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto issue = [&](int64_t t, int s) {
    const Gemv1ManyMat& M = a.m[mat_of(t)];
    const int r0 = (int)(t - M.tile0) * a.R, nr = min(a.R, M.d_out - r0);
    const unsigned bytes = (unsigned)(nr * a.row_bytes);
    mbar_expect_tx(&bar[s], bytes);
    bulk_g2s(stage + (size_t)s * a.stage_bytes, M.packed + (int64_t)r0 * a.row_bytes, bytes, &bar[s]);
  };
  if (tid == 0) {
    for (int s = 0; s < kGemvManyStages && t_lo + s < t_hi; ++s) {
      issue(t_lo + s, s);
      issued[s] = 1;
    }
  }
  const int sl = warp % a.S, kk = warp / a.S;
  const int c = sl * 32 + lane;
  const bool active = c < C;
  const uint32_t copy = (uint32_t)lane & (uint32_t)(copies - 1);
  float xr[kE];
  int cur = -1;
  int flags = 0;
  int it = 0;
  for (int64_t t = t_lo; t < t_hi; ++t, ++it) {
    const int st = it % kGemvManyStages;
    if (!mbar_wait_bounded(&bar[st], (unsigned)(it / kGemvManyStages) & 1u)) {
      flags |= QAMW_STATUS_TIMEOUT;
      break;
    }
    const int mi = mat_of(t);
    const Gemv1ManyMat& M = a.m[mi];
    if (mi != cur) {  // this lane's chunk of the matrix's x_bar
      cur = mi;
      if (active) {
        const float4* xp = reinterpret_cast<const float4*>(M.xbar + (int64_t)c * kE);
#pragma unroll
        for (int q = 0; q < kE / 4; ++q) {
          const float4 f = __ldg(xp + q);
          xr[4 * q] = f.x;
          xr[4 * q + 1] = f.y;
          xr[4 * q + 2] = f.z;
          xr[4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kE; ++j) xr[j] = 0.f;
      }
    }
    const int r0 = (int)(t - M.tile0) * a.R, nr = min(a.R, M.d_out - r0);
    const unsigned char* buf = stage + (size_t)st * a.stage_bytes;
    float* part = partial + st * part_floats;
    for (int rl = kk; rl < nr; rl += a.k) {
      float acc0 = 0.f, acc1 = 0.f;
      if (active) {
        const uint32_t* src =
            reinterpret_cast<const uint32_t*>(buf + (size_t)rl * a.row_bytes) + (size_t)c * BITS;
        uint32_t w[BITS];
#pragma unroll
        for (int q = 0; q < BITS; ++q) w[q] = src[q];
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
        M.y[r0 + r] = __float2bfloat16_rn(sum * __half2float(M.rnorm[r0 + r]));
      }
      __syncwarp();
      if (lane == 0) {
        done[st] = 0;
        if (t + kGemvManyStages < t_hi) {
          issue(t + kGemvManyStages, st);
          issued[st] += 1;
        }
      }
    }
  }
  // after a timeout: let the copies still in flight land before this CTA's
  // shared memory goes away
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < kGemvManyStages; ++s)
      if (issued[s] > 0) mbar_wait_bounded(&bar[s], (unsigned)(issued[s] - 1) & 1u);
  }
  raise_flag(a.status, flags);
}

// One run: x_bar of its matrices, then their products.
template <int BITS>
cudaError_t run_gemv1_many(const qamw_matrix* const* ms, int n, const uint16_t* const* xs,
                           uint16_t* const* ys, float* const* xbars, int32_t* d_status,
                           cudaStream_t stream) {
  const qamw_matrix& f = *ms[0];
  {
    Xbar1Args<kGemvManyMax> xa;
    for (int i = 0; i < n; ++i) {
      xa.m[i].x = reinterpret_cast<const __nv_bfloat16*>(xs[i]);
      xa.m[i].sigma = reinterpret_cast<const __half*>(ms[i]->sigma);
      xa.m[i].scale = reinterpret_cast<const __half*>(ms[i]->chan_scale);
      xa.m[i].xbar = xbars[i];
      xa.m[i].seed = ms[i]->mask_seed;
    }
    xa.status = d_status;
    xa.n = n;
    xa.d_in = f.d_in;
    xa.block = f.block;
    const int64_t V = (int64_t)n * (f.d_in / kE);
    cudaError_t err = launch_pdl(k_xbar1_many<kGemvManyMax>,
                                 dim3((unsigned)((V + kXb1Threads - 1) / kXb1Threads)),
                                 dim3(kXb1Threads), 0, stream, xa);
    if (err != cudaSuccess) return err;
  }
  Gemv1ManyArgs<kGemvManyMax> a;
  a.codebook = reinterpret_cast<const float2*>(f.codebook);
  a.status = d_status;
  a.row_bytes = f.row_bytes;
  a.n = n;
  a.d_in = f.d_in;
  a.K = 1 << f.bits;
  const int C = f.d_in / kE;
  a.S = (C + 31) / 32;
  a.k = a.S <= 16 ? 16 / a.S : 1;  // 16 warps (512 threads) per SM
  int R = (int)(kGemvManyTileBytes / f.row_bytes);
  R = R < a.k ? a.k : (R / a.k) * a.k;
  a.R = R;
  a.stage_bytes = (unsigned)(R * f.row_bytes);
  int64_t tiles = 0;
  for (int i = 0; i < n; ++i) {
    a.m[i].packed = ms[i]->packed;
    a.m[i].rnorm = reinterpret_cast<const __half*>(ms[i]->row_norm);
    a.m[i].xbar = xbars[i];
    a.m[i].y = reinterpret_cast<__nv_bfloat16*>(ys[i]);
    a.m[i].tile0 = tiles;
    a.m[i].d_out = ms[i]->d_out;
    tiles += (ms[i]->d_out + R - 1) / R;
  }
  a.ntiles = tiles;
  int cl = a.K <= 1024 ? 5 : 4;
  while (cl > 0 && gemv1_many_smem(a.K, cl, a.stage_bytes, R, a.S) > 227 * 1024) --cl;
  a.copies_log2 = cl;
  const size_t smem = gemv1_many_smem(a.K, cl, a.stage_bytes, R, a.S);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  const int threads = 32 * a.S * a.k;
  const void* fn = threads <= 256
                       ? reinterpret_cast<const void*>(&k_gemv1_many<BITS, 256, kGemvManyMax>)
                       : reinterpret_cast<const void*>(&k_gemv1_many<BITS, 512, kGemvManyMax>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  if (threads <= 256)
    return launch_pdl(k_gemv1_many<BITS, 256, kGemvManyMax>, dim3(grid), dim3(threads), smem,
                      stream, a);
  return launch_pdl(k_gemv1_many<BITS, 512, kGemvManyMax>, dim3(grid), dim3(threads), smem, stream,
                    a);
}

// ------------------------------------------------------------- batch 2..16

constexpr int kRotItems = 32;
constexpr int kRotThreads = 256;

// ------------------------------------------------------ tensor-core path
//
// y^T = C_hat x_bar^T on the tensor cores with m16n8k16 MMAs and fp32
// accumulation: A = 16 rows x 16 k of gathered codewords (one k pair = one
// codeword (x, y)), B = 16 k x 8 batch columns of x_bar, C = 16 rows x 8
// columns.  Both operands are split into binary16 high and low parts (v = hi +
// lo, lo = binary16(v - hi)) and C accumulates A_hi B_hi + A_lo B_hi + A_hi B_lo:
// about 22 significant bits, where a single binary16 operand would spend most of
// the 1e-2 tolerance on rows whose output is small.
// The order of the k dimension makes each lane's A operands one whole
// 64-column chunk of a row: in K-chunk j (128 pairs, 16 k-steps), k-step kk,
// lane (g = lane / 4, t = lane % 4) holds pairs p0 = 128 j + 32 t + 2 kk (k
// slots 2t, 2t+1) and p0 + 1 (slots 2t+8, 2t+9) of rows g and g + 8 -- its
// indices are the `bits` words of chunk 4 j + t, extracted with fixed shifts.
// B uses the same order: the rotation kernel writes x_bar in it.
constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = 32 * kMmaWarps;
constexpr int kMmaRows = 16;       // rows per CTA tile
constexpr int kMmaPairs = 128;     // pairs per K-chunk
constexpr int kMmaStages = 2;

__host__ __device__ inline int mma_chunks(int P) { return (P + kMmaPairs - 1) / kMmaPairs; }

// Bytes of x_bar in the tensor-core layout: [chunk][n-tile][kk][lane] uint4
// {hi(x_bar_n[p]), hi(x_bar_n[p + 1]), lo(x_bar_n[p]), lo(x_bar_n[p + 1])}
// (binary16 pairs), n = 8 nt + g, p = 128 j + 32 t + 2 kk; zero for n >= batch
// and p >= P.
__host__ __device__ inline size_t mma_xbar_bytes(int P, int NT) {
  return (size_t)mma_chunks(P) * NT * 16 * 32 * sizeof(uint4);
}

// Codeword replicas (log2) of the hi/lo table (8 bytes an entry): 8 for K =
// 2048, 16 below (at most 128 KB).
constexpr int mma_rep_log2(int bits) { return bits >= 11 ? 3 : 4; }

// binary16 high and low parts of a pair of floats, as two half2 words.
__device__ __forceinline__ uint2 split_half2(float a, float b) {
  const __half2 hi = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(hi);
  const __half2 lo = __floats2half2_rn(a - hf.x, b - hf.y);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
}

// x_bar = sigma (.) R_fwd(x / s) for n < 8 NT columns and every 64-column
// chunk (padded to whole K-chunks), written in the tensor-core layout.  A CTA
// takes 32 (column, chunk) items: all threads form D x / s element by element
// into shared memory, then one warp rotates the 32 chunks (lane = item).
__global__ void __launch_bounds__(kRotThreads) k_rotate_mma(const __nv_bfloat16* __restrict__ x,
                                                            int batch, int NT, int d_in, int block,
                                                            uint64_t seed,
                                                            const __half* __restrict__ s,
                                                            const __half* __restrict__ sigma,
                                                            uint4* __restrict__ xb,
                                                            int32_t* status) {
  __shared__ float buf[kRotItems][kE + 1];  // +1: conflict-free rows and columns
  const int C = d_in / kE;
  const int Cpad = mma_chunks(d_in / 2) * 4;
  const int ncol = 8 * NT;
  const int64_t V = (int64_t)ncol * Cpad;
  const int nb = min(block, kE), lanes = max(block / kE, 1);
  const float inv_sqrt_b = 1.0f / sqrtf((float)block);
  int flags = 0;
  // s and sigma may come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  for (int64_t base = (int64_t)blockIdx.x * kRotItems; base < V;
       base += (int64_t)gridDim.x * kRotItems) {
    // item v = n Cpad + c: the b / 64 chunks of a Hadamard block are
    // consecutive items, inside one CTA's 32 (Cpad and 32 are multiples of
    // b / 64), and padding chunks c >= C form whole blocks of zeros
    for (int e = threadIdx.x; e < kRotItems * kE; e += kRotThreads) {
      const int i = e / kE, j = e - i * kE;
      const int64_t v = base + i;
      const int64_t n = v < V ? v / Cpad : ncol;
      float val = 0.f;
      if (n < batch) {
        const int c = (int)(v - n * Cpad);
        if (c < C) {
          const int col = c * kE + j;
          const float xv = __bfloat162float(x[n * d_in + col]);
          if (!isfinite(xv)) flags |= QAMW_STATUS_NONFINITE;
          const float q = __fdiv_rn(xv, __half2float(s[col]));
          val = mask_negative(seed, (uint32_t)col) ? -q : q;
        }
      }
      buf[i][j] = val;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // one whole warp: the lane shuffles need all 32
      const int64_t v = base + threadIdx.x;
      const bool active = v < V;
      const int64_t n = active ? v / Cpad : 0;
      const int c = active ? (int)(v - n * Cpad) : 0;
      float xv[kE];
#pragma unroll
      for (int j = 0; j < kE; ++j) xv[j] = buf[threadIdx.x][j];
      fwht_reg<kE>(xv, nb);
      fwht_lanes<kE>(xv, lanes);
      if (active) {
        float sg[kQ];
        if (c < C && n < batch) {
          load_halves<kQ>(sigma + (int64_t)c * kQ, sg);
        } else {
#pragma unroll
          for (int q = 0; q < kQ; ++q) sg[q] = 0.f;
        }
        const int jc = c >> 2, tt = c & 3, nt = (int)(n >> 3), g = (int)(n & 7);
        uint4* dst = xb + ((size_t)(jc * NT + nt) * 16) * 32 + 4 * g + tt;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const float f0 = sg[2 * kk] * inv_sqrt_b, f1 = sg[2 * kk + 1] * inv_sqrt_b;
          const float a = xv[4 * kk] * f0, b = xv[4 * kk + 1] * f0;
          const float cc = xv[4 * kk + 2] * f1, d = xv[4 * kk + 3] * f1;
          if (fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(cc), fabsf(d))) > 65504.f)
            flags |= QAMW_STATUS_RANGE;
          const uint2 p0 = split_half2(a, b), p1 = split_half2(cc, d);
          dst[kk * 32] = make_uint4(p0.x, p1.x, p0.y, p1.y);
        }
      }
    }
    __syncthreads();
  }
  raise_flag(status, flags);
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

struct GemvMmaArgs {
  const uint8_t* packed;
  const __half* rnorm;
  const float2* codebook;
  const uint4* xb;
  __nv_bfloat16* y;
  int32_t* status;
  int64_t row_bytes;
  int d_out, P, batch, K;
};

// Shared memory: table uint2 [K][replicas] | per warp ring [2][16 rows][16 bits
// bytes] | red float [8 warps][16 rows][8 NT] | bars [8][2].
size_t gemv_mma_smem(int K, int bits, int NT) {
  return ((size_t)K << (mma_rep_log2(bits) + 3)) +
         (size_t)kMmaWarps * kMmaStages * kMmaRows * 16 * bits +
         (size_t)kMmaWarps * kMmaRows * 8 * NT * sizeof(float) + kMmaWarps * kMmaStages * 8;
}

// The CTA takes 16-row tiles tile = blockIdx.x, + gridDim.x, ...; warp w takes
// K-chunks w, w + 8, ... of each.  The warp's (tile, chunk) items stream their
// 16 row segments (16 bits bytes each) through the warp's own 2-stage ring of
// bulk copies, one copy per lane, prefetching across tiles.  The 8 warps'
// partial sums of a tile are added in a fixed order.
template <int BITS, int NT>
__global__ void __launch_bounds__(kMmaThreads, 1) k_gemv_mma(const GemvMmaArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int RL = mma_rep_log2(BITS);
  constexpr unsigned kSeg = 16u * BITS;  // bytes of one row segment of a chunk
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  uint2* tab = reinterpret_cast<uint2*>(smem);
  unsigned char* ring = smem + ((size_t)a.K << (RL + 3)) + (size_t)warp * kMmaStages * kMmaRows * kSeg;
  float* red = reinterpret_cast<float*>(smem + ((size_t)a.K << (RL + 3)) +
                                        (size_t)kMmaWarps * kMmaStages * kMmaRows * kSeg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + kMmaWarps * kMmaRows * 8 * NT) + warp * kMmaStages;
  // the codeword table needs nothing from the kernels ahead
  for (int j = tid; j < a.K; j += kMmaThreads) {
    const float2 c = __ldg(a.codebook + j);
    const uint2 u = split_half2(c.x, c.y);
#pragma unroll
    for (int r = 0; r < (1 << RL); ++r) tab[(j << RL) + ((r + lane) & ((1 << RL) - 1))] = u;
  }
  if (lane == 0) {
    for (int s = 0; s < kMmaStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // x_bar, the indices and r_hat come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  const uint32_t tab_s = smem_u32(tab);
  const uint32_t rep8 = (uint32_t)(lane & ((1 << RL) - 1)) << 3;
  const int nchunks = mma_chunks(a.P);
  const int ntiles = (a.d_out + kMmaRows - 1) / kMmaRows;
  const int my_tiles = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int nmy = warp < nchunks ? (nchunks - warp + kMmaWarps - 1) / kMmaWarps : 0;
  const int nitems = my_tiles * nmy;  // this warp's (tile, chunk) items
  const unsigned used = (unsigned)a.row_bytes;
  unsigned issued = 0;  // lane 0: bit s = stage s had a copy; bit 8 + s = its last phase
  int flags = 0;
  bool abort = false;
  auto issue = [&](int i) {  // item i: one row segment per lane
    const int tile = blockIdx.x + (i / nmy) * gridDim.x;
    const int j = warp + (i % nmy) * kMmaWarps;
    const int row0 = tile * kMmaRows, nrows = min(kMmaRows, a.d_out - row0);
    const unsigned st = (unsigned)i % kMmaStages;
    const unsigned bytes = min(kSeg, used - (unsigned)j * kSeg);
    if (lane == 0) {
      mbar_expect_tx(&bars[st], bytes * (unsigned)nrows);
      issued = (issued & (1u << st)) ? (issued ^ (1u << (8 + st))) : (issued | (1u << st));
    }
    __syncwarp();
    if (lane < nrows)
      bulk_g2s(ring + (st * kMmaRows + lane) * kSeg,
               a.packed + (int64_t)(row0 + lane) * a.row_bytes + (int64_t)j * kSeg, bytes, &bars[st]);
  };
  for (int i = 0; i < min(kMmaStages, nitems); ++i) issue(i);
  int item = 0;
  for (int ti = 0; ti < my_tiles; ++ti) {
    const int tile = blockIdx.x + ti * gridDim.x;
    const int row0 = tile * kMmaRows, nrows = min(kMmaRows, a.d_out - row0);
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    for (int ci = 0; ci < nmy && !abort; ++ci, ++item) {
      const int j = warp + ci * kMmaWarps;
      const unsigned st = (unsigned)item % kMmaStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], ((unsigned)item / kMmaStages) & 1u))) {
        flags |= QAMW_STATUS_TIMEOUT;
        abort = true;
        break;
      }
      uint32_t wa[BITS], wb[BITS];
      {
        const uint32_t* s0 = reinterpret_cast<const uint32_t*>(ring + (st * kMmaRows + g) * kSeg) + t * BITS;
        const uint32_t* s1 = reinterpret_cast<const uint32_t*>(ring + (st * kMmaRows + g + 8) * kSeg) + t * BITS;
#pragma unroll
        for (int w = 0; w < BITS; ++w) {
          wa[w] = s0[w];
          wb[w] = s1[w];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (item + kMmaStages < nitems) issue(item + kMmaStages);
      const uint4* xbj = a.xb + ((size_t)j * NT * 16) * 32 + lane;
      uint32_t ia[kQ], ib[kQ];
      unpack32<BITS>(wa, ia);
      unpack32<BITS>(wb, ib);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const uint2 a0 = lds_u2(tab_s + ((ia[2 * kk] << (RL + 3)) | rep8));
        const uint2 a1 = lds_u2(tab_s + ((ib[2 * kk] << (RL + 3)) | rep8));
        const uint2 a2 = lds_u2(tab_s + ((ia[2 * kk + 1] << (RL + 3)) | rep8));
        const uint2 a3 = lds_u2(tab_s + ((ib[2 * kk + 1] << (RL + 3)) | rep8));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 b = __ldg(xbj + (nt * 16 + kk) * 32);
          mma_16816(acc[nt], a0.x, a1.x, a2.x, a3.x, b.x, b.y);  // hi . hi
          mma_16816(acc[nt], a0.y, a1.y, a2.y, a3.y, b.x, b.y);  // lo . hi
          mma_16816(acc[nt], a0.x, a1.x, a2.x, a3.x, b.z, b.w);  // hi . lo
        }
      }
    }
    // partial sums of this warp: rows g, g + 8; columns 8 nt + 2 t, + 1
    float* rw = red + (size_t)warp * kMmaRows * 8 * NT;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      rw[g * 8 * NT + 8 * nt + 2 * t] = acc[nt][0];
      rw[g * 8 * NT + 8 * nt + 2 * t + 1] = acc[nt][1];
      rw[(g + 8) * 8 * NT + 8 * nt + 2 * t] = acc[nt][2];
      rw[(g + 8) * 8 * NT + 8 * nt + 2 * t + 1] = acc[nt][3];
    }
    if (__syncthreads_or(abort)) break;
    for (int e = tid; e < kMmaRows * a.batch; e += kMmaThreads) {
      const int r = e % kMmaRows, n = e / kMmaRows;
      if (r >= nrows) continue;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kMmaWarps; ++w) sum += red[(size_t)w * kMmaRows * 8 * NT + r * 8 * NT + n];
      a.y[(int64_t)n * a.d_out + row0 + r] = __float2bfloat16_rn(sum * __half2float(a.rnorm[row0 + r]));
    }
    __syncthreads();  // red is rewritten by the next tile
  }
  // copies still in flight (after a timeout) land before shared memory goes away
  if (lane == 0) {
    for (int s = 0; s < kMmaStages; ++s)
      if (issued & (1u << s)) mbar_wait_bounded(&bars[s], (issued >> (8 + s)) & 1u);
  }
  raise_flag(a.status, flags);
}

template <int BITS, int NT>
cudaError_t run_gemv_mma(const qamw_matrix& m, int batch, const uint4* xb, uint16_t* d_y,
                         int32_t* d_status, cudaStream_t stream) {
  GemvMmaArgs a;
  a.packed = m.packed;
  a.rnorm = reinterpret_cast<const __half*>(m.row_norm);
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.xb = xb;
  a.y = reinterpret_cast<__nv_bfloat16*>(d_y);
  a.status = d_status;
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.P = m.d_in / 2;
  a.batch = batch;
  a.K = 1 << m.bits;
  const size_t smem = gemv_mma_smem(a.K, BITS, NT);
  const void* fn = reinterpret_cast<const void*>(&k_gemv_mma<BITS, NT>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int ntiles = (m.d_out + kMmaRows - 1) / kMmaRows;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  return launch_pdl(k_gemv_mma<BITS, NT>, dim3(grid), dim3(kMmaThreads), smem, stream, a);
}

cudaError_t rotate_mma(const qamw_matrix& m, const uint16_t* d_x, int batch, int NT, uint4* xb,
                       int32_t* d_status, cudaStream_t stream) {
  const int64_t V = (int64_t)8 * NT * mma_chunks(m.d_in / 2) * 4;
  const void* fn = reinterpret_cast<const void*>(&k_rotate_mma);
  const int grid = persistent_grid(fn, kRotThreads, 0, (V + kRotItems - 1) / kRotItems);
  return launch_pdl(k_rotate_mma, dim3(grid), dim3(kRotThreads), 0, stream,
                    reinterpret_cast<const __nv_bfloat16*>(d_x), batch, NT, m.d_in, m.block,
                    m.mask_seed, reinterpret_cast<const __half*>(m.chan_scale),
                    reinterpret_cast<const __half*>(m.sigma), xb, d_status);
}

template <int BITS>
cudaError_t gemv_bits(const qamw_matrix& m, const uint16_t* d_x, int batch, const float2* xbar,
                      uint16_t* d_y, int32_t* d_status, cudaStream_t stream) {
  if (batch == 1) return run_gemv1<BITS>(m, d_x, d_y, d_status, stream);
  // batch 2..16: rotation into the tensor-core layout, then the MMA kernel
  uint4* xb = reinterpret_cast<uint4*>(const_cast<float2*>(xbar));
  const int NT = batch <= 8 ? 1 : 2;
  cudaError_t err = rotate_mma(m, d_x, batch, NT, xb, d_status, stream);
  if (err != cudaSuccess) return err;
  return NT == 1 ? run_gemv_mma<BITS, 1>(m, batch, xb, d_y, d_status, stream)
                 : run_gemv_mma<BITS, 2>(m, batch, xb, d_y, d_status, stream);
}

}  // namespace

size_t gemv_workspace_bytes(int d_in, int batch) {
  // x_bar of batch > 1 in the tensor-core layout (8 or 16 columns, whole
  // K-chunks); never less than 16 columns of fp32 pairs
  (void)batch;
  const size_t mma = mma_xbar_bytes(d_in / 2, 2);
  const size_t f32 = (size_t)16 * (size_t)(d_in / 2) * sizeof(float2);
  return mma > f32 ? mma : f32;
}

cudaError_t launch_decode_gemv(const qamw_matrix& m, const uint16_t* d_x, int batch,
                               uint16_t* d_y, void* d_ws, int32_t* d_status,
                               cudaStream_t stream) {
  float2* xbar = static_cast<float2*>(d_ws);
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

size_t gemv_many_workspace_bytes(const qamw_matrix* ms, int n) {
  size_t b = 0;
  for (int i = 0; i < n; ++i)
    if (ms[i].d_out > 0) b += ((size_t)ms[i].d_in * sizeof(float) + 255) & ~(size_t)255;
  return b;
}

cudaError_t launch_decode_gemv_many(const qamw_matrix* ms, int n, const uint16_t* const* d_x,
                                    uint16_t* const* d_y, void* d_ws, int32_t* d_status,
                                    cudaStream_t stream) {
  // runs of up to kGemvManyMax consecutive matrices with the same d_in, block,
  // bits and codebook; x_bar of matrix i at its offset in the workspace
  std::vector<const qamw_matrix*> g;
  std::vector<const uint16_t*> gx;
  std::vector<uint16_t*> gy;
  std::vector<float*> gb;
  auto flush = [&]() -> cudaError_t {
    if (g.empty()) return cudaSuccess;
    cudaError_t e;
    switch (g[0]->bits) {
#define QAMW_GEMV_MANY_CASE(B)                                                                 \
  case B:                                                                                     \
    e = run_gemv1_many<B>(g.data(), (int)g.size(), gx.data(), gy.data(), gb.data(), d_status, \
                          stream);                                                            \
    break;
      QAMW_GEMV_MANY_CASE(1) QAMW_GEMV_MANY_CASE(2) QAMW_GEMV_MANY_CASE(3) QAMW_GEMV_MANY_CASE(4)
      QAMW_GEMV_MANY_CASE(5) QAMW_GEMV_MANY_CASE(6) QAMW_GEMV_MANY_CASE(7) QAMW_GEMV_MANY_CASE(8)
      QAMW_GEMV_MANY_CASE(9) QAMW_GEMV_MANY_CASE(10) QAMW_GEMV_MANY_CASE(11)
#undef QAMW_GEMV_MANY_CASE
      default: e = cudaErrorInvalidValue;
    }
    g.clear();
    gx.clear();
    gy.clear();
    gb.clear();
    return e;
  };
  unsigned char* ws = static_cast<unsigned char*>(d_ws);
  for (int i = 0; i < n; ++i) {
    if (ms[i].d_out == 0) continue;
    if (!g.empty()) {
      const qamw_matrix& f = *g[0];
      if (f.d_in != ms[i].d_in || f.block != ms[i].block || f.bits != ms[i].bits ||
          f.codebook != ms[i].codebook || (int)g.size() == kGemvManyMax) {
        const cudaError_t e = flush();
        if (e != cudaSuccess) return e;
      }
    }
    g.push_back(&ms[i]);
    gx.push_back(d_x[i]);
    gy.push_back(d_y[i]);
    gb.push_back(reinterpret_cast<float*>(ws));
    ws += ((size_t)ms[i].d_in * sizeof(float) + 255) & ~(size_t)255;
  }
  return flush();
}

}  // namespace qamw
