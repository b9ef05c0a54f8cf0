// encode.cu -- QAM-W encoder (paper section 3.1 steps 1-6, section 3.4, and the
// activation-aware per-channel scaling).
//
// The channel scales and eq. (1) come first (calibrate.cu); then
//   k_encode        norm, rotate, normalise, nearest codeword, pack  (row groups)
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

// ---------------------------------------------------------------- encoder

template <typename T>
struct EncodeArgs {
  const T* W;
  const __half* scale;
  const __half* sigma;
  const float2* codebook;
  const void* prefilter;  // nullable: exhaustive search
  uint8_t* packed;
  __half* rnorm;
  int32_t* status;
  unsigned long long* candidates;  // nullable: codewords scored, summed
  int64_t row_bytes;
  int d_out, d_in, block, K;
  int rows_per_cta;  // R: whole rows per CTA iteration, R * C <= blockDim
  int hs_side;       // k_encode: inner-grid cells per side copied to shared memory
  int hs_gi;         // k_encode: inner-grid size the launch was sized for
  uint64_t seed;
};

// One CTA iteration encodes R whole rows; thread (r, c) owns chunk c of row r.
// Steps 1-6 of section 3.1 in one pass over W: scale by s, sum of squares
// (reduced per row in a fixed order, so r is bitwise reproducible), Hadamard
// butterflies, division by r sqrt(b) and sigma_k, nearest codeword, packing.
// This form searches straight from the 64 rotated values in registers; it
// serves rows too wide for k_encode's shared-memory point buffer.
template <int BITS, typename T, int MODE>
__global__ void __launch_bounds__(512, 1) k_encode_wide(const EncodeArgs<T> a) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  float2* cb2 = reinterpret_cast<float2*>(smem);
  // per-column tables transposed, [position in chunk][chunk], so that the lanes
  // of a warp (consecutive chunks) read consecutive words
  const int P = a.d_in >> 1, C = a.d_in / kE;
  float* fT = reinterpret_cast<float*>(cb2 + ((a.K + 1) & ~1));  // [j][c]: D * s of column 64c + j
  float* isgT = fT + a.d_in;                        // [q][c]: 1 / sigma of pair 32c + q
  float* part = isgT + P;                           // [blockDim] partial sums of squares
  float* rsum = part + blockDim.x;                  // [R] row norms
  // polar: amplitude levels a_i = codeword (i Np).x of the expanded table;
  // scalar: levels l_i = codeword (i L).x of the product table
  constexpr int kBa = BITS / 2, kNa = 1 << kBa, kNp = 1 << (BITS - kBa);
  float* lev = reinterpret_cast<float*>(cb2);
  if constexpr (MODE != kJointMode) {
    for (int i = threadIdx.x; i < kNa; i += blockDim.x) lev[i] = a.codebook[i * kNp].x;
  } else {
    // table fills: unrolled so that each thread's loads are in flight together
#pragma unroll 4
    for (int i = threadIdx.x; i < a.K; i += blockDim.x) cb2[i] = a.codebook[i];
  }
  const uint64_t seed = a.seed;
  fill_interleaved<kE>(fT, a.scale, a.d_in, C, [=](int j, float v) {
    return mask_negative(seed, (uint32_t)j) ? -v : v;
  });
  fill_interleaved<kQ>(isgT, a.sigma, P, C, [](int, float v) { return 1.0f / v; });
  PrefilterView pf;
  if (a.prefilter != nullptr) {
    pf = prefilter_view(a.prefilter, a.K);
  } else {
    pf.G = 0;
    pf.Gf = 0.f;
    pf.R = 0.f;
    pf.inv_h = 0.f;
  }
  __syncthreads();

  const int R = a.rows_per_cta;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int rl = threadIdx.x / C, c = threadIdx.x - rl * C;
  const int nb = min(a.block, kE), lanes = max(a.block / kE, 1);
  const float sqrt_b = sqrtf((float)a.block);
  int flags = 0;
  unsigned scored = 0;
  const bool count = a.candidates != nullptr;
  for (int64_t r0 = (int64_t)blockIdx.x * R; r0 < a.d_out; r0 += (int64_t)gridDim.x * R) {
    const int64_t row = r0 + rl;
    const bool active = rl < R && row < a.d_out;
    float x[kE];
    float ss = 0.f;
    if (active) {
      load64(a.W + row * a.d_in + (int64_t)c * kE, x);
#pragma unroll
      for (int j = 0; j < kE; ++j) {
        x[j] *= fT[j * C + c];
        ss = fmaf(x[j], x[j], ss);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kE; ++j) x[j] = 0.f;
    }
    part[threadIdx.x] = ss;
    fwht_reg<kE>(x, nb);
    fwht_lanes<kE>(x, lanes);
    __syncthreads();
    for (int q = warp; q < R; q += nwarps) {
      float t = 0.f;
      for (int k = lane; k < C; k += 32) t += part[q * C + k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) rsum[q] = sqrtf(t);
    }
    __syncthreads();
    if (!active) continue;

    const float r = rsum[rl];
    if (c == 0) {
      const __half h = __float2half_rn(r);
      a.rnorm[row] = h;
      if (!isfinite(r)) flags |= QAMW_STATUS_NONFINITE;
      else if (isinf(__half2float(h))) flags |= QAMW_STATUS_RANGE;
    }
    const bool zero = !(r > 0.f) || !isfinite(r);  // zero or not finite (flagged): indices 0
    const float inv = 1.0f / (r * sqrt_b);
    // nearest codeword of each pair, packing as we go; the list head of pair
    // q+1 is fetched while pair q is scored
    uint32_t w[BITS];
#pragma unroll
    for (int t = 0; t < BITS; ++t) w[t] = 0u;
    if constexpr (MODE != kJointMode) {
      const float np_over_2pi = (float)kNp * 0.159154943f;
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float f = inv * isgT[q * C + c];
        const float px = x[2 * q] * f, py = x[2 * q + 1] * f;
        const uint32_t id =
            zero ? 0u
                 : (uint32_t)(MODE == kPolarMode ? polar_index(px, py, lev, kNa, kNp, np_over_2pi)
                                                 : scalar_index(px, py, lev, kNa));
        scored += kNa;
        const int bit = q * BITS, wi = bit >> 5, sh = bit & 31;
        w[wi] |= id << sh;
        if (sh + BITS > 32) w[wi + 1] |= id >> (32 - sh);
      }
    } else {
      const float f0 = inv * isgT[c];
      float px = x[0] * f0, py = x[1] * f0;
      uint2 cur = pf_head(px, py, pf);
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        float nx = 0.f, ny = 0.f;
        uint2 nxt = cur;
        if (q + 1 < kQ) {
          const float f1 = inv * isgT[(q + 1) * C + c];
          nx = x[2 * q + 2] * f1;
          ny = x[2 * q + 3] * f1;
          nxt = pf_head(nx, ny, pf);
        }
        const uint32_t id =
            zero ? 0u : (uint32_t)pf_finish2(cur, px, py, cb2, a.K, pf, scored, count);
        const int bit = q * BITS, wi = bit >> 5, sh = bit & 31;
        w[wi] |= id << sh;
        if (sh + BITS > 32) w[wi + 1] |= id >> (32 - sh);
        cur = nxt;
        px = nx;
        py = ny;
      }
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.packed + row * a.row_bytes) + (size_t)c * BITS;
#pragma unroll
    for (int t = 0; t < BITS; ++t) dst[t] = w[t];
    if (c == C - 1) {  // zero the row's padding words
      for (int64_t o = (int64_t)C * BITS * 4; o < a.row_bytes; o += 4)
        *reinterpret_cast<uint32_t*>(a.packed + row * a.row_bytes + o) = 0u;
    }
  }
  raise_flag(a.status, flags);
  if (a.candidates != nullptr) {
    unsigned long long v = scored;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) atomicAdd(a.candidates, v);
  }
}

// The same steps with the list heads in shared memory.  One CTA of R rows x C
// chunk-threads (at most 512 threads, one CTA per SM).  Each row's C threads
// synchronise on the row's own named barrier when C is a multiple of 32 (so
// that rows drift apart and one row's search overlaps another's loads), else
// on the CTA barrier.  Per row:
//   load, scale, sum of squares, butterflies; the row norm (every warp of the
//   row reduces the row's partial sums in one fixed order, so r is bitwise
//   reproducible);
//   then in two halves of 16 pairs: normalise into the thread's own column of
//   the point buffer and search those points in a rolled loop (the list head of
//   point q + 2 is fetched while point q is scored), packing the indices
//   through a 64-bit bit accumulator that emits each 32-bit word as it fills.
// List heads come from a shared copy of the central S x S cells of the table's
// inner grid (filled by bulk copies while the other tables are built); points
// outside it, or whose inner list is longer than a head, read the main table.
// Shared memory: cb2 float2[K] | fT4 float4[16][C] | isg4 float4[8][C] |
// part float[2][T] | rsum float[R] (padded) | pts float2[16][T] | hs uint2[S][S]
// | bar uint64.
template <int BITS, typename T, int MODE>
__global__ void __launch_bounds__(512, 1) k_encode(const EncodeArgs<T> a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int C = a.d_in / kE, NT = blockDim.x, R = a.rows_per_cta;
  float2* cb2 = reinterpret_cast<float2*>(smem);
  float4* fT4 = reinterpret_cast<float4*>(smem + (((size_t)a.K * sizeof(float2) + 15) & ~15));
  float4* isg4 = fT4 + (kE / 4) * C;
  float* part = reinterpret_cast<float*>(isg4 + (kQ / 4) * C);  // [2][NT]
  float* rsum = part + 2 * NT;                                   // [R], padded to 16 bytes
  float2* pts = reinterpret_cast<float2*>(rsum + ((R + 3) & ~3));  // [16][NT]
  uint2* hs = reinterpret_cast<uint2*>(pts + (size_t)(kQ / 2) * NT);  // [S][S]
  uint64_t* bar = reinterpret_cast<uint64_t*>(hs + (size_t)a.hs_side * a.hs_side);

  PrefilterView pf;
  if (a.prefilter != nullptr) {
    pf = prefilter_view(a.prefilter, a.K);
  } else {
    pf.G = 0;
    pf.Gf = 0.f;
    pf.R = 0.f;
    pf.inv_h = 0.f;
    pf.Gi = 0;
  }
  // the shared copy of the inner grid: its table must be the one the launch
  // was sized for (a table for another codebook size reads as none)
  const int S = (MODE == kJointMode && pf.G > 0 && pf.Gi == a.hs_gi) ? a.hs_side : 0;
  const int c0 = (pf.Gi - S) / 2;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (S > 0) {
    if (threadIdx.x == 0) mbar_expect_tx(bar, (unsigned)(S * S * 8));
    for (int r = threadIdx.x; r < S; r += NT)
      bulk_g2s(hs + (size_t)r * S, pf.inner + (size_t)(c0 + r) * pf.Gi + c0, (unsigned)(S * 8), bar);
  }
  // polar: amplitude levels a_i = codeword (i Np).x of the expanded table;
  // scalar: levels l_i = codeword (i L).x of the product table
  constexpr int kBa = BITS / 2, kNa = 1 << kBa, kNp = 1 << (BITS - kBa);
  float* lev = reinterpret_cast<float*>(cb2);
  if constexpr (MODE != kJointMode) {
    for (int i = threadIdx.x; i < kNa; i += NT) lev[i] = a.codebook[i * kNp].x;
  } else {
#pragma unroll 4
    for (int i = threadIdx.x; i < a.K; i += NT) cb2[i] = a.codebook[i];
  }
  pdl_wait();  // s and sigma below, W, and the outputs, after the kernel ahead
  pdl_trigger();
  const uint64_t seed = a.seed;
  fill_quads<kE>(fT4, a.scale, a.d_in, C, [=](int j, float v) {
    return mask_negative(seed, (uint32_t)j) ? -v : v;
  });
  fill_quads<kQ>(isg4, a.sigma, a.d_in / 2, C, [](int, float v) { return 1.0f / v; });
  __syncthreads();
  int flags = 0;
  // the head copy is waited for just before a thread's first search, so that it
  // overlaps the first row's loads and butterflies; a thread whose wait runs out
  // searches the main table instead (same results) and flags TIMEOUT
  int S_eff = S;
  bool hs_pending = S > 0;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = NT >> 5;
  const int rl = threadIdx.x / C, c = threadIdx.x - rl * C;
  const bool per_row = (C % 32) == 0;  // a row is whole warps: it has its own barrier
  const int nb = min(a.block, kE), lanes = max(a.block / kE, 1);
  const float sqrt_b = sqrtf((float)a.block);
  const bool count = a.candidates != nullptr;
  float2* mypts = pts + threadIdx.x;
  unsigned scored = 0;
  int buf = 0;
  // this CTA's rows: a contiguous block of floor or ceil(d_out / grid)
  const int64_t row_lo = (int64_t)blockIdx.x * a.d_out / gridDim.x;
  const int64_t row_hi = ((int64_t)blockIdx.x + 1) * a.d_out / gridDim.x;
  for (int64_t r0 = row_lo; r0 < row_hi; r0 += R) {
    const int64_t row = r0 + rl;
    const bool active = rl < R && row < row_hi;
    if (per_row && !active) continue;  // the row's threads all skip, barrier included
    float x[kE];
    float ss = 0.f;
    if (active) {
      if (c == 0 && row + R < row_hi)  // this thread group's next row, into L2
        bulk_prefetch_l2(a.W + (row + R) * a.d_in, (unsigned)(a.d_in * (int64_t)sizeof(T)));
      load64(a.W + row * a.d_in + (int64_t)c * kE, x);
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
    float* pb = part + buf * NT;
    buf ^= 1;
    pb[threadIdx.x] = ss;
    fwht_reg<kE>(x, nb);
    fwht_lanes<kE>(x, lanes);
    float r;
    if (per_row) {
      // the row's partial sums: double-buffered, so one barrier per row suffices
      asm volatile("bar.sync %0, %1;" ::"r"(1 + rl), "r"(C) : "memory");
      float t = 0.f;
      for (int k = lane; k < C; k += 32) t += pb[rl * C + k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      r = sqrtf(t);
    } else {
      __syncthreads();
      for (int q = warp; q < R; q += nwarps) {
        float t = 0.f;
        for (int k = lane; k < C; k += 32) t += pb[q * C + k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0) rsum[q] = sqrtf(t);
      }
      __syncthreads();
      if (!active) continue;
      r = rsum[rl];
    }

    if (c == 0) {
      const __half h = __float2half_rn(r);
      a.rnorm[row] = h;
      if (!isfinite(r)) flags |= QAMW_STATUS_NONFINITE;
      else if (isinf(__half2float(h))) flags |= QAMW_STATUS_RANGE;
    }
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.packed + row * a.row_bytes) + (size_t)c * BITS;
    const float inv = 1.0f / (r * sqrt_b);
    // zero row, not finite (flagged), or a norm so small that 1 / (r sqrt(b))
    // overflows (points that would not be finite): every index 0
    if (!(r > 0.f) || !isfinite(r) || !isfinite(inv)) {
#pragma unroll
      for (int t = 0; t < BITS; ++t) dst[t] = 0u;
    } else {
      if (hs_pending) {
        hs_pending = false;
        if (!mbar_wait_bounded(bar, 0)) {
          S_eff = 0;
          flags |= QAMW_STATUS_TIMEOUT;
        }
      }
      // each index goes to the first word of its point's slot once the point
      // has been read; the 16 indices of a half are then packed with fixed
      // shifts (LSB first, index k at bits [k BITS, (k + 1) BITS))
      uint32_t* myid = reinterpret_cast<uint32_t*>(mypts);
      uint32_t w[BITS];
#pragma unroll
      for (int t = 0; t < BITS; ++t) w[t] = 0u;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        // normalise pairs 16 hf .. 16 hf + 15 into the point buffer
#pragma unroll
        for (int i = 0; i < kQ / 8; ++i) {
          const float4 is = isg4[(hf * (kQ / 8) + i) * C + c];
          const int q0 = hf * (kQ / 2) + 4 * i;
          // p_k = z_k / sigma_k with z = y / (r sqrt(b)): one factor per pair
          const float f0 = inv * is.x, f1 = inv * is.y, f2 = inv * is.z, f3 = inv * is.w;
          mypts[(4 * i + 0) * NT] = make_float2(x[2 * q0 + 0] * f0, x[2 * q0 + 1] * f0);
          mypts[(4 * i + 1) * NT] = make_float2(x[2 * q0 + 2] * f1, x[2 * q0 + 3] * f1);
          mypts[(4 * i + 2) * NT] = make_float2(x[2 * q0 + 4] * f2, x[2 * q0 + 5] * f2);
          mypts[(4 * i + 3) * NT] = make_float2(x[2 * q0 + 6] * f3, x[2 * q0 + 7] * f3);
        }
        if constexpr (MODE != kJointMode) {
          const float np_over_2pi = (float)kNp * 0.159154943f;
#pragma unroll 4
          for (int q = 0; q < kQ / 2; ++q) {
            const float2 p = mypts[q * NT];
            myid[q * 2 * NT] =
                (uint32_t)(MODE == kPolarMode ? polar_index(p.x, p.y, lev, kNa, kNp, np_over_2pi)
                                              : scalar_index(p.x, p.y, lev, kNa));
            scored += kNa;
          }
        } else {
          // the list heads of points q + 2, q + 3 are fetched while q, q + 1
          // are scored; a resolved point's slot becomes (index, ~0), a point
          // that needs the full search keeps its slot and is found below
          const uint32_t cb_s = smem_u32(cb2);
          uint32_t rare = 0;
          float2 p = mypts[0];
          uint2 ha = pf_head_shared(p.x, p.y, pf, hs, S_eff, c0);
          p = mypts[NT];
          uint2 hb = pf_head_shared(p.x, p.y, pf, hs, S_eff, c0);
#pragma unroll 1
          for (int q = 0; q < kQ / 2; q += 2) {
            p = mypts[min(q + 2, kQ / 2 - 1) * NT];
            const uint2 hc = pf_head_shared(p.x, p.y, pf, hs, S_eff, c0);
            p = mypts[min(q + 3, kQ / 2 - 1) * NT];
            const uint2 hd = pf_head_shared(p.x, p.y, pf, hs, S_eff, c0);
            p = mypts[q * NT];
            uint32_t id = pf_finish_fast(ha, p.x, p.y, cb_s, scored, count);
            rare |= id;
            if (id != kPfRare) reinterpret_cast<uint2*>(mypts)[q * NT] = make_uint2(id, ~0u);
            p = mypts[(q + 1) * NT];
            id = pf_finish_fast(hb, p.x, p.y, cb_s, scored, count);
            rare |= id;
            if (id != kPfRare) reinterpret_cast<uint2*>(mypts)[(q + 1) * NT] = make_uint2(id, ~0u);
            ha = hc;
            hb = hd;
          }
          // points off the grid, lists longer than a head, or no list
          if (__any_sync(__activemask(), (rare >> 31) != 0u)) {
#pragma unroll 1
            for (int k = 0; k < kQ / 2; ++k) {
              const uint2 v = reinterpret_cast<const uint2*>(mypts)[k * NT];
              if (v.y != ~0u)
                myid[k * 2 * NT] = (uint32_t)nearest_pf2(__uint_as_float(v.x), __uint_as_float(v.y),
                                                         cb2, a.K, pf, scored, count);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < kQ / 2; ++k) {
          const uint32_t id = myid[k * 2 * NT];
          const int bit = (hf * (kQ / 2) + k) * BITS, wi = bit >> 5, sh = bit & 31;
          w[wi] |= id << sh;
          if (sh + BITS > 32) w[wi + 1] |= id >> (32 - sh);
        }
      }
#pragma unroll
      for (int t = 0; t < BITS; ++t) dst[t] = w[t];
    }
    if (c == C - 1) {  // zero the row's padding words
      for (int64_t o = (int64_t)C * BITS * 4; o < a.row_bytes; o += 4)
        *reinterpret_cast<uint32_t*>(a.packed + row * a.row_bytes + o) = 0u;
    }
  }
  if (S > 0 && threadIdx.x == 0) mbar_wait_bounded(bar, 0);  // no copy in flight at exit
  raise_flag(a.status, flags);
  if (a.candidates != nullptr) {
    unsigned long long v = scored;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) atomicAdd(a.candidates, v);
  }
}

// The normalised points p_k = z_k / sigma_k of rows [row0, row0 + nrows)
// (section 3.1 steps 1-4): the encoder's first phase, with the same fixed-order
// row-norm reduction and the same p = y (1 / (r sqrt(b)) (1 / sigma_k)), so the
// points are bitwise those the encoder searches.  Rows whose norm is zero or
// not finite give NaN points.  out: float2 [nrows][d_in / 2].
template <typename T>
__global__ void __launch_bounds__(512) k_points(const EncodeArgs<T> a, int64_t row0,
                                                int64_t nrows, float2* __restrict__ out) {
  extern __shared__ __align__(16) float psm[];
  const int P = a.d_in >> 1, C = a.d_in / kE, R = a.rows_per_cta;
  float* fT = psm;          // [j][c]: D * s of column 64c + j
  float* isgT = fT + a.d_in;  // [q][c]: 1 / sigma of pair 32c + q
  float* part = isgT + P;   // [blockDim]
  float* rsum = part + blockDim.x;
  const uint64_t seed = a.seed;
  fill_interleaved<kE>(fT, a.scale, a.d_in, C, [=](int j, float v) {
    return mask_negative(seed, (uint32_t)j) ? -v : v;
  });
  fill_interleaved<kQ>(isgT, a.sigma, P, C, [](int, float v) { return 1.0f / v; });
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int rl = threadIdx.x / C, c = threadIdx.x - rl * C;
  const int nb = min(a.block, kE), lanes = max(a.block / kE, 1);
  const float sqrt_b = sqrtf((float)a.block);
  int flags = 0;
  for (int64_t g0 = (int64_t)blockIdx.x * R; g0 < nrows; g0 += (int64_t)gridDim.x * R) {
    const int64_t g = g0 + rl;  // row within the range
    const bool active = rl < R && g < nrows;
    float x[kE];
    float ss = 0.f;
    if (active) {
      load64(a.W + (row0 + g) * a.d_in + (int64_t)c * kE, x);
#pragma unroll
      for (int j = 0; j < kE; ++j) {
        x[j] *= fT[j * C + c];
        ss = fmaf(x[j], x[j], ss);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kE; ++j) x[j] = 0.f;
    }
    part[threadIdx.x] = ss;
    fwht_reg<kE>(x, nb);
    fwht_lanes<kE>(x, lanes);
    __syncthreads();
    for (int q = warp; q < R; q += nwarps) {
      float t = 0.f;
      for (int k = lane; k < C; k += 32) t += part[q * C + k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) rsum[q] = sqrtf(t);
    }
    __syncthreads();
    if (!active) continue;
    const float r = rsum[rl];
    if (!isfinite(r)) flags |= QAMW_STATUS_NONFINITE;
    const bool none = !(r > 0.f) || !isfinite(r);
    const float inv = 1.0f / (r * sqrt_b);
    float4* dst = reinterpret_cast<float4*>(out + g * P + (int64_t)c * kQ);
#pragma unroll
    for (int q = 0; q < kQ; q += 2) {
      const float f0 = inv * isgT[q * C + c], f1 = inv * isgT[(q + 1) * C + c];
      dst[q / 2] = none ? make_float4(NAN, NAN, NAN, NAN)
                        : make_float4(x[2 * q] * f0, x[2 * q + 1] * f0, x[2 * q + 2] * f1,
                                      x[2 * q + 3] * f1);
    }
  }
  raise_flag(a.status, flags);
}

// Rows per CTA iteration and the CTA size for k_encode_wide: R whole rows of C
// chunk-threads, R * C <= 512, chosen so that few threads idle and the CTA has
// 128-512 threads.
void encode_shape(int C, int* R_out, int* threads_out) {
  int bestR = 1, bestT = ((C + 31) / 32) * 32;
  double bestScore = -1.0;
  for (int R = 1; R * C <= 512; ++R) {
    const int T = ((R * C + 31) / 32) * 32;
    const double eff = (double)(R * C) / T;
    // prefer 256-thread CTAs: two per SM at <= 128 registers
    const double score = eff - (T < 256 ? 0.05 * (256 - T) / 128.0 : 0.0) - (T > 256 ? 0.02 : 0.0);
    if (score > bestScore + 1e-9) {
      bestScore = score;
      bestR = R;
      bestT = T;
    }
  }
  *R_out = bestR;
  *threads_out = bestT;
}

// k_encode's shape: R rows of C chunk-threads (at most 15 rows -- one named
// barrier each -- and 512 threads, one CTA per SM) and the side S of the shared
// copy of the inner grid, the largest multiple of 4 that fits next to the other
// tables (at most the inner grid).  Returns false when the tables and the
// point buffer alone do not fit (very wide rows: k_encode_wide).
bool encode_shared_shape(int C, int K, int d_in, int gi, int* R_out, int* threads_out,
                         int* side_out, size_t* smem_out) {
  const int R = std::max(1, std::min(15, 512 / C));
  const int T = ((R * C + 31) / 32) * 32;
  const size_t base = (((size_t)K * sizeof(float2) + 15) & ~(size_t)15) +
                      (size_t)d_in * sizeof(float) + (size_t)(d_in / 2) * sizeof(float) +
                      2 * (size_t)T * sizeof(float) + (size_t)((R + 3) & ~3) * sizeof(float) +
                      (size_t)(kQ / 2) * T * sizeof(float2) + sizeof(uint64_t);
  const size_t cap = 227 * 1024;
  if (R * C > 512 || base > cap) return false;
  int S = (int)std::sqrt((double)(cap - base) / 8.0);
  S = std::min(S, gi) & ~3;
  if (S < 8) S = 0;
  *R_out = R;
  *threads_out = T;
  *side_out = S;
  *smem_out = base + (size_t)S * S * 8;
  return true;
}

template <int BITS, typename T, int MODE>
cudaError_t run_encode(EncodeArgs<T> a, cudaStream_t stream) {
  const int C = a.d_in / kE;
  const int gi = (a.prefilter != nullptr && MODE == kJointMode) ? prefilter_inner(prefilter_grid(BITS)) : 0;
  int R, threads, side = 0;
  size_t smem;
  const void* fn;
  if (encode_shared_shape(C, a.K, a.d_in, gi, &R, &threads, &side, &smem)) {
    fn = reinterpret_cast<const void*>(&k_encode<BITS, T, MODE>);
  } else {
    encode_shape(C, &R, &threads);
    smem = (size_t)((a.K + 1) & ~1) * sizeof(float2) + (size_t)a.d_in * sizeof(float) +
           (size_t)(a.d_in / 2) * sizeof(float) + (size_t)threads * sizeof(float) +
           (size_t)R * sizeof(float);
    fn = reinterpret_cast<const void*>(&k_encode_wide<BITS, T, MODE>);
  }
  a.rows_per_cta = R;
  a.hs_side = side;
  a.hs_gi = gi;
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(fn, threads, smem, (a.d_out + R - 1) / R);
  void* args[] = {&a};
  return launch_pdl_ptr(fn, dim3(grid), dim3(threads), smem, stream, args);
}

template <typename T, int MODE>
cudaError_t encode_rows_typed(const T* W, const qamw_matrix& m, int32_t* st,
                              unsigned long long* cand, cudaStream_t stream) {
  EncodeArgs<T> a;
  a.W = W;
  a.scale = reinterpret_cast<const __half*>(m.chan_scale);
  a.sigma = reinterpret_cast<const __half*>(m.sigma);
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.prefilter = m.prefilter;
  a.packed = m.packed;
  a.rnorm = reinterpret_cast<__half*>(m.row_norm);
  a.status = st;
  a.candidates = cand;
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.d_in = m.d_in;
  a.block = m.block;
  a.K = 1 << m.bits;
  a.rows_per_cta = 1;
  a.hs_side = 0;
  a.hs_gi = 0;
  a.seed = m.mask_seed;
  switch (m.bits) {
    case 1: return run_encode<1, T, MODE>(a, stream);
    case 2: return run_encode<2, T, MODE>(a, stream);
    case 3: return run_encode<3, T, MODE>(a, stream);
    case 4: return run_encode<4, T, MODE>(a, stream);
    case 5: return run_encode<5, T, MODE>(a, stream);
    case 6: return run_encode<6, T, MODE>(a, stream);
    case 7: return run_encode<7, T, MODE>(a, stream);
    case 8: return run_encode<8, T, MODE>(a, stream);
    case 9: return run_encode<9, T, MODE>(a, stream);
    case 10: return run_encode<10, T, MODE>(a, stream);
    case 11: return run_encode<11, T, MODE>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

// Section 3.5: Lloyd-Max levels of the unit Rayleigh density on one warp (lane
// i owns level i, Na <= 32), fp64, from the equal-probability thresholds, then
// the expanded table c[ia Np + ip] = a_ia (cos 2 pi ip / Np, sin 2 pi ip / Np).
__global__ void __launch_bounds__(32) k_polar_codebook(int bits, int iters, float2* __restrict__ cb) {
  const int ba = bits / 2, Na = 1 << ba, Np = 1 << (bits - ba);
  const int i = threadIdx.x;
  const double rt2 = 1.4142135623730950488, c = 1.2533141373155002512;  // sqrt 2, sqrt(pi/2)
  auto lower = [&](int k) { return k == 0 ? 0.0 : sqrt(-2.0 * log(1.0 - (double)k / Na)); };
  double t0 = lower(i), t1 = i + 1 < Na ? lower(i + 1) : INFINITY;
  double lv = 0.0;
  for (int it = 0; it <= iters; ++it) {
    // centroid of [t0, t1): (t0 e0 - t1 e1 + c (erf(t1/rt2) - erf(t0/rt2))) / (e0 - e1)
    const double e0 = exp(-0.5 * t0 * t0);
    const double e1 = isinf(t1) ? 0.0 : exp(-0.5 * t1 * t1);
    const double te1 = isinf(t1) ? 0.0 : t1 * e1;
    const double erf1 = isinf(t1) ? 1.0 : erf(t1 / rt2);
    lv = (t0 * e0 - te1 + c * (erf1 - erf(t0 / rt2))) / (e0 - e1);
    if (it == iters) break;
    const double below = __shfl_up_sync(0xffffffffu, lv, 1);
    const double above = __shfl_down_sync(0xffffffffu, lv, 1);
    if (i > 0 && i < Na) t0 = 0.5 * (below + lv);
    if (i + 1 < Na) t1 = 0.5 * (lv + above);
  }
  if (i < Na) {
    for (int ip = 0; ip < Np; ++ip) {
      const double phi = 6.283185307179586477 * ip / Np;
      cb[i * Np + ip] = make_float2((float)(lv * cos(phi)), (float)(lv * sin(phi)));
    }
  }
}

// The d = 1 ablation (paper section 2, parallel work): Lloyd-Max levels of
// N(0, 1) on one warp (lane i owns level i, L = 2^(bits/2) <= 32), fp64, from
// thresholds evenly spaced on [-3, 3]; then the product table
// c[ix L + iy] = (l_ix, l_iy).
__global__ void __launch_bounds__(32) k_scalar_codebook(int bits, int iters, float2* __restrict__ cb) {
  const int L = 1 << (bits / 2);
  const int i = threadIdx.x;
  const double rt2 = 1.4142135623730950488, inv_sqrt2pi = 0.39894228040143267794;
  double t0 = i == 0 ? -INFINITY : -3.0 + 6.0 * i / L;
  double t1 = i + 1 < L ? -3.0 + 6.0 * (i + 1) / L : INFINITY;
  double lv = 0.0;
  for (int it = 0; it <= iters; ++it) {
    // centroid of [t0, t1): (phi(t0) - phi(t1)) / (Phi(t1) - Phi(t0))
    const double p0 = isinf(t0) ? 0.0 : inv_sqrt2pi * exp(-0.5 * t0 * t0);
    const double p1 = isinf(t1) ? 0.0 : inv_sqrt2pi * exp(-0.5 * t1 * t1);
    const double e0 = isinf(t0) ? -1.0 : erf(t0 / rt2);
    const double e1 = isinf(t1) ? 1.0 : erf(t1 / rt2);
    lv = (p0 - p1) / (0.5 * (e1 - e0));
    if (it == iters) break;
    const double below = __shfl_up_sync(0xffffffffu, lv, 1);
    const double above = __shfl_down_sync(0xffffffffu, lv, 1);
    if (i > 0 && i < L) t0 = 0.5 * (below + lv);
    if (i + 1 < L) t1 = 0.5 * (lv + above);
  }
  for (int j = 0; j < L; ++j) {
    const double lj = __shfl_sync(0xffffffffu, lv, j);
    if (i < L) cb[j * L + i] = make_float2((float)lj, (float)lv);
  }
}

}  // namespace

cudaError_t launch_polar_codebook(int bits, float* d_codebook, cudaStream_t stream) {
  k_polar_codebook<<<1, 32, 0, stream>>>(bits, 20000, reinterpret_cast<float2*>(d_codebook));
  return cudaGetLastError();
}

cudaError_t launch_scalar_codebook(int bits, float* d_codebook, cudaStream_t stream) {
  k_scalar_codebook<<<1, 32, 0, stream>>>(bits, 20000, reinterpret_cast<float2*>(d_codebook));
  return cudaGetLastError();
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t encode_workspace_bytes(int d_out, int d_in, int bits, EncodeWorkspace* carve, void* base) {
  const size_t off = calibrate_workspace_bytes(d_out, d_in, carve, base);
  if (carve) carve->prefilter = static_cast<char*>(base) + off;
  return off + align256(prefilter_bytes_for(prefilter_grid(bits)));
}

template <typename T>
cudaError_t points_typed(const T* W, const qamw_matrix& m, int64_t row0, int64_t nrows,
                         float2* out, int32_t* st, cudaStream_t stream) {
  EncodeArgs<T> a{};
  a.W = W;
  a.scale = reinterpret_cast<const __half*>(m.chan_scale);
  a.sigma = reinterpret_cast<const __half*>(m.sigma);
  a.status = st;
  a.d_out = m.d_out;
  a.d_in = m.d_in;
  a.block = m.block;
  a.seed = m.mask_seed;
  const int C = m.d_in / kE;
  const int R = std::max(1, 256 / C);
  a.rows_per_cta = R;
  const int threads = ((R * C + 31) / 32) * 32;
  const size_t smem = (size_t)m.d_in * 4 + (size_t)(m.d_in / 2) * 4 + (size_t)threads * 4 +
                      (size_t)R * 4;
  const void* fn = reinterpret_cast<const void*>(&k_points<T>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(fn, threads, smem, (nrows + R - 1) / R);
  k_points<T><<<grid, threads, smem, stream>>>(a, row0, nrows, out);
  return cudaGetLastError();
}

cudaError_t launch_points(const void* d_W, int dtype, const qamw_matrix& m, int64_t row0,
                          int64_t nrows, float* d_points, int32_t* d_status, cudaStream_t stream) {
  float2* out = reinterpret_cast<float2*>(d_points);
  if (dtype == QAMW_DTYPE_BF16)
    return points_typed(static_cast<const __nv_bfloat16*>(d_W), m, row0, nrows, out, d_status,
                        stream);
  return points_typed(static_cast<const float*>(d_W), m, row0, nrows, out, d_status, stream);
}

cudaError_t launch_encode_rows(const void* d_W, int dtype, const qamw_matrix& m, int32_t* d_status,
                               unsigned long long* d_candidates, int mode, cudaStream_t stream) {
  const bool f32 = dtype == QAMW_DTYPE_F32;
  const float* Wf = static_cast<const float*>(d_W);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(d_W);
  switch (mode) {
    case kPolarMode:
      return f32 ? encode_rows_typed<float, kPolarMode>(Wf, m, d_status, d_candidates, stream)
                 : encode_rows_typed<__nv_bfloat16, kPolarMode>(Wb, m, d_status, d_candidates, stream);
    case kScalarMode:
      return f32 ? encode_rows_typed<float, kScalarMode>(Wf, m, d_status, d_candidates, stream)
                 : encode_rows_typed<__nv_bfloat16, kScalarMode>(Wb, m, d_status, d_candidates, stream);
    default:
      return f32 ? encode_rows_typed<float, kJointMode>(Wf, m, d_status, d_candidates, stream)
                 : encode_rows_typed<__nv_bfloat16, kJointMode>(Wb, m, d_status, d_candidates, stream);
  }
}

cudaError_t launch_encode(const void* d_W, int dtype, const float* d_act_stat, float alpha,
                          int flags, const qamw_matrix& m, const EncodeWorkspace& ws,
                          int32_t* d_status, cudaStream_t stream) {
  cudaError_t err;
  if (!(flags & QAMW_SCALES_GIVEN)) {
    err = launch_channel_scales(d_act_stat, m.d_in, alpha, m.chan_scale, d_status, stream);
    if (err != cudaSuccess) return err;
  }
  if (!(flags & QAMW_SIGMA_GIVEN)) {
    err = launch_calibrate(d_W, dtype, m, ws, d_status, stream);
    if (err != cudaSuccess) return err;
  }
  if (flags & QAMW_POLAR)
    return launch_encode_rows(d_W, dtype, m, d_status, nullptr, kPolarMode, stream);
  if (flags & QAMW_SCALAR)
    return launch_encode_rows(d_W, dtype, m, d_status, nullptr, kScalarMode, stream);
  qamw_matrix mm = m;
  if (mm.prefilter == nullptr) {
    err = launch_build_prefilter(m.codebook, m.bits, prefilter_grid(m.bits), ws.prefilter, stream);
    if (err != cudaSuccess) return err;
    mm.prefilter = ws.prefilter;
  }
  return launch_encode_rows(d_W, dtype, mm, d_status, nullptr, kJointMode, stream);
}

}  // namespace qamw
