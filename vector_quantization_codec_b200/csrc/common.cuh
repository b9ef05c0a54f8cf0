// common.cuh -- device helpers shared by the QAM-W kernels (sm_100a).
//
// Thread layout used by every row kernel: a row of d_in columns is cut into
// chunks of kE = 64 consecutive columns (kQ = 32 pairs); one thread owns one
// (row, chunk).  Virtual thread v = row * C + chunk, C = d_in / 64, runs as
// thread v % blockDim of a grid-stride loop, so lane = v % 32.  A Hadamard
// block of b > 64 columns spans b/64 consecutive chunks = b/64 consecutive,
// aligned lanes (C is a multiple of b/64), and the butterflies across chunks
// are warp shuffles; blocks of b <= 64 columns stay inside one thread.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qamw.h"

namespace qamw {

constexpr int kE = 64;  // columns per thread chunk
constexpr int kQ = 32;  // pairs per thread chunk
// Largest d_in: the encoder keeps 6 bytes per column (D_j s_j and 1/sigma) plus
// a 32 KB codebook in shared memory, within the 227 KB a CTA may use.
constexpr int kMaxDin = 32768;

// splitmix64 (Steele, Lea & Flood; Vigna's formulation) evaluated at a counter.
__device__ __forceinline__ uint64_t mix64(uint64_t counter) {
  uint64_t z = counter + 0x9e3779b97f4a7c15ULL;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

// Sign of column j in the deterministic mask D: negative when bit 63 is set.
__device__ __forceinline__ bool mask_negative(uint64_t seed, uint32_t j) {
  return (mix64((seed << 32) + j) >> 63) != 0;
}

__device__ __forceinline__ void raise_flag(int32_t* status, int flag) {
  if (flag && status) atomicOr(status, flag);
}

// One butterfly stage of span H over N values held in registers.
template <int N, int H>
__device__ __forceinline__ void fwht_stage(float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; i += 2 * H) {
#pragma unroll
    for (int j = i; j < i + H; ++j) {
      const float a = v[j], b = v[j + H];
      v[j] = a + b;
      v[j + H] = a - b;
    }
  }
}

// Sylvester Hadamard butterflies of span < nb over the N values a thread holds
// (N and nb powers of two).  With nb >= N this is v <- H_N v in natural order;
// with nb < N it is H_nb on each group of nb consecutive values.  The stages
// are expanded at compile time so that v stays in registers.
template <int N, int H = 1>
__device__ __forceinline__ void fwht_reg(float (&v)[N], int nb) {
  if constexpr (H < N) {
    if (H < nb) fwht_stage<N, H>(v);
    fwht_reg<N, 2 * H>(v, nb);
  }
}

// Remaining butterflies of a block that spans `lanes` consecutive lanes
// (H_lanes applied across the lanes' chunks).  All 32 lanes must call it.
template <int N>
__device__ __forceinline__ void fwht_lanes(float (&v)[N], int lanes) {
  const unsigned lane = threadIdx.x & 31u;
  for (int s = 1; s < lanes; s <<= 1) {
    const bool upper = (lane & (unsigned)s) != 0;
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, v[j], s);
      v[j] = upper ? (o - v[j]) : (v[j] + o);
    }
  }
}

// 32 indices of BITS bits from BITS little-endian 32-bit words (LSB first).
template <int BITS>
__device__ __forceinline__ void unpack32(const uint32_t (&w)[BITS], uint32_t (&idx)[kQ]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    const int bit = q * BITS, wi = bit >> 5, sh = bit & 31;
    uint32_t v;
    if (sh + BITS <= 32)
      v = w[wi] >> sh;
    else
      v = __funnelshift_r(w[wi], w[wi + 1], sh);
    idx[q] = v & mask;
  }
}

// Index q (compile-time) of the 32 packed in w.
template <int BITS, int Q>
__device__ __forceinline__ uint32_t extract_idx(const uint32_t (&w)[BITS]) {
  constexpr int bit = Q * BITS, wi = bit >> 5, sh = bit & 31;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  if constexpr (sh + BITS <= 32)
    return (w[wi] >> sh) & mask;
  else
    return __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
}

template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&idx)[kQ], uint32_t (&w)[BITS]) {
#pragma unroll
  for (int t = 0; t < BITS; ++t) w[t] = 0u;
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    const int bit = q * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] |= idx[q] << sh;
    if (sh + BITS > 32) w[wi + 1] |= idx[q] >> (32 - sh);
  }
}

// 64 consecutive weights of type T as fp32.
__device__ __forceinline__ void load64(const float* p, float (&x)[kE]) {
  const float4* s = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int t = 0; t < kE / 4; ++t) {
    const float4 v = __ldg(s + t);
    x[4 * t] = v.x;
    x[4 * t + 1] = v.y;
    x[4 * t + 2] = v.z;
    x[4 * t + 3] = v.w;
  }
}

__device__ __forceinline__ void load64(const __nv_bfloat16* p, float (&x)[kE]) {
  const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int t = 0; t < kE / 8; ++t) {
    const uint4 v = __ldg(s + t);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * t + 2 * e] = __uint_as_float(u[e] << 16);
      x[8 * t + 2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
    }
  }
}

// n consecutive binary16 values (n a multiple of 8, 16-byte aligned) as fp32,
// with all loads issued before any use.
template <int N>
__device__ __forceinline__ void load_halves(const __half* p, float (&x)[N]) {
  uint4 v[N / 8];
  const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int t = 0; t < N / 8; ++t) v[t] = __ldg(s + t);
#pragma unroll
  for (int t = 0; t < N / 8; ++t) {
    const __half2* h = reinterpret_cast<const __half2*>(&v[t]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h[e]);
      x[8 * t + 2 * e] = f.x;
      x[8 * t + 2 * e + 1] = f.y;
    }
  }
}

// Cooperative fill of a chunk-interleaved table: dst[(j % PERIOD) * C + j / PERIOD]
// = f(j, src[j]) for j < n, src binary16 (16-byte aligned, n a multiple of 8),
// 8 values per 16-byte load, every thread's loads issued together.
template <int PERIOD, typename F>
__device__ __forceinline__ void fill_interleaved(float* dst, const __half* src, int n, int C,
                                                 F f) {
#pragma unroll 2
  for (int j8 = threadIdx.x * 8; j8 < n; j8 += blockDim.x * 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + j8));
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f2 = __half22float2(h[e]);
      const int j = j8 + 2 * e;
      dst[(j % PERIOD) * C + j / PERIOD] = f(j, f2.x);
      dst[((j + 1) % PERIOD) * C + (j + 1) / PERIOD] = f(j + 1, f2.y);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------- async bulk copies
// cp.async.bulk global -> shared with mbarrier completion (TMA, no tensor map,
// never multicast).  Every wait is bounded: kSpinLimit tries with a short sleep
// between them (well under a second in total) before the caller gives up.
constexpr unsigned kSpinLimit = 1u << 20;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// src and dst 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}" : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity) {
  for (unsigned i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    __nanosleep(256);
  }
  return false;
}

// ---------------------------------------------------------------- prefilter
// Table written by the prefilter kernels and read by the encoder / trainer.
struct PrefilterHeader {
  float R;       // grid covers [-R, R)^2
  float inv_h;   // G / (2R)
  float h;       // cell side
  float margin;  // squared-distance slack for fp32 rounding in the encoder
  int32_t G;     // cells per side (0: no grid, always exhaustive)
  int32_t cap;   // list capacity per cell
  int32_t K;
  int32_t NS;    // angular sectors for points off the grid (|p| >= R)
};

// Each cell's (or sector's) list: the count and the candidate indices in
// ascending order.  It is stored twice:
//   head (8 bytes, one per list, all heads side by side): bits 0-3 hold
//     min(count, 15) -- 15 meaning "15 or more, or overflowed: see the tail" --
//     and bits 4-63 five 12-bit candidate slots; slots past the count repeat
//     the first candidate.  One 8-byte load resolves almost every point, and
//     a 128-byte line holds 16 neighbouring heads.
//   tail (64 bytes): 32 uint16 slots, slot 0 the exact count (kPfOverflow:
//     search exhaustively), slots 1..count the candidates.
constexpr int kPfSlots = 32;
constexpr int kPfCap = kPfSlots - 1;         // candidates per list
constexpr uint32_t kPfOverflow = 0xffffu;
constexpr int kPfHeadSlots = 5;

__host__ __device__ inline int prefilter_grid(int bits) {
  return bits <= 5 ? 0 : (bits <= 7 ? 64 : (bits <= 9 ? 128 : 256));
}

__host__ __device__ inline size_t prefilter_lists_offset() {
  return (sizeof(PrefilterHeader) + 15) / 16 * 16;
}

// Points off the grid are looked up by angle in kPfSectors equal sectors of
// the region |p| >= R (list of every codeword that can win there).
constexpr int kPfSectors = 256;

__host__ __device__ inline int prefilter_sectors(int bits) {
  return prefilter_grid(bits) > 0 ? kPfSectors : 0;
}

__host__ __device__ inline size_t prefilter_bytes_for(int bits) {
  const size_t n = (size_t)prefilter_grid(bits) * prefilter_grid(bits) + prefilter_sectors(bits);
  return prefilter_lists_offset() + ((n * 8 + 15) / 16) * 16 + n * kPfSlots * sizeof(uint16_t);
}

// List n (cells 0..G*G-1, then sectors): head at heads[n] (8 bytes), tail at
// tails[n] (32 uint16).
__host__ __device__ inline size_t prefilter_tails_offset(size_t nlists) {
  return prefilter_lists_offset() + ((nlists * 8 + 15) / 16) * 16;
}

struct PrefilterView {
  float R, inv_h, Gf;
  int G;  // 0: exhaustive search only
  int NS;
  const uint2* heads;     // [G*G + NS]
  const uint16_t* tails;  // [G*G + NS][32]
};

// A table built for another codebook size is ignored (exhaustive search), so a
// list entry can never index past the K codewords in shared memory.
__device__ __forceinline__ PrefilterView prefilter_view(const void* table, int K) {
  const PrefilterHeader* h = reinterpret_cast<const PrefilterHeader*>(table);
  PrefilterView v;
  v.R = h->R;
  v.inv_h = h->inv_h;
  v.G = (h->K == K && h->cap == kPfCap && h->NS == kPfSectors) ? h->G : 0;
  v.NS = h->NS;
  v.Gf = (float)v.G;
  const size_t nlists = (size_t)h->G * h->G + h->NS;
  v.heads = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(table) +
                                           prefilter_lists_offset());
  v.tails = reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(table) +
                                              prefilter_tails_offset(nlists));
  return v;
}

// Codeword j in shared memory as (x, y, x^2 + y^2, 0).  The nearest codeword of
// p minimises |c|^2 - 2 p.c (= |p - c|^2 - |p|^2), two FMAs per candidate.
__device__ __forceinline__ float4 codeword_q(float2 c) {
  return make_float4(c.x, c.y, fmaf(c.x, c.x, c.y * c.y), 0.f);
}

// Exhaustive search, ascending j with a strict '<' (lowest index on ties).
// `scored` accumulates the number of codewords evaluated.
__device__ __forceinline__ int nearest_all(float m2x, float m2y, const float4* cbq, int K,
                                           unsigned& scored) {
  scored += (unsigned)K;
  float be = INFINITY;
  int bi = 0;
  for (int j = 0; j < K; ++j) {
    const float4 c = cbq[j];
    const float e = fmaf(m2x, c.x, fmaf(m2y, c.y, c.z));
    if (e < be) {
      be = e;
      bi = j;
    }
  }
  return bi;
}

__device__ __forceinline__ void score(float m2x, float m2y, const float4* cbq, uint32_t j,
                                      float& be, int& bi) {
  const float4 c = cbq[j];
  const float e = fmaf(m2x, c.x, fmaf(m2y, c.y, c.z));
  if (e < be) {
    be = e;
    bi = (int)j;
  }
}

// Split form of nearest_pf, so that a caller can fetch the next point's list
// head while it scores the current point.
struct PfCursor {
  const uint16_t* tail;  // nullptr: exhaustive search
  uint2 head;
};

__device__ __forceinline__ PfCursor pf_locate(float px, float py, const PrefilterView& pf) {
  PfCursor cur;
  cur.tail = nullptr;
  cur.head = make_uint2(0u, 0u);
  if (pf.G > 0 && isfinite(px) && isfinite(py)) {
    const float gx = (px + pf.R) * pf.inv_h;
    const float gy = (py + pf.R) * pf.inv_h;
    size_t n;
    if (gx >= 0.f && gx < pf.Gf && gy >= 0.f && gy < pf.Gf) {
      n = (size_t)((int)gy * pf.G + (int)gx);
    } else {
      const float t = (atan2f(py, px) + 3.14159265f) * ((float)pf.NS * 0.159154943f);
      n = (size_t)pf.G * pf.G + min(max((int)t, 0), pf.NS - 1);
    }
    cur.head = __ldg(pf.heads + n);
    cur.tail = pf.tails + n * kPfSlots;
  }
  return cur;
}

// Rare paths of pf_finish: lists longer than the 5 head slots (tail slots
// 6..count), overflowed lists and points that are not finite (exhaustive
// search).  Kept out of line so that the common path stays small.
static __device__ __noinline__ int pf_finish_slow(const uint16_t* tail, float m2x, float m2y,
                                                  const float4* cbq, int K, float be, int bi,
                                                  unsigned* scored) {
  const uint32_t cnt = tail == nullptr ? kPfOverflow : (uint32_t)__ldg(tail);
  if (cnt == kPfOverflow) return nearest_all(m2x, m2y, cbq, K, *scored);
  *scored += cnt - kPfHeadSlots;
  for (uint32_t t = kPfHeadSlots + 1; t <= cnt; ++t) score(m2x, m2y, cbq, __ldg(tail + t), be, bi);
  return bi;
}

// The 5 head slots are always filled (unused ones repeat the first candidate,
// which cannot change a strict-'<' argmin taken in ascending slot order), so
// the common case scores 5 codewords without branching.
__device__ __forceinline__ int pf_finish(const PfCursor& cur, float px, float py,
                                         const float4* cbq, int K, unsigned& scored) {
  const float m2x = -2.f * px, m2y = -2.f * py;
  const uint2 h = cur.head;
  const uint32_t n5 = h.x & 15u;
  float be = INFINITY;
  int bi = 0;
  if (cur.tail != nullptr) {
    score(m2x, m2y, cbq, (h.x >> 4) & 0xfffu, be, bi);
    score(m2x, m2y, cbq, (h.x >> 16) & 0xfffu, be, bi);
    score(m2x, m2y, cbq, (h.x >> 28) | ((h.y & 0xffu) << 4), be, bi);
    score(m2x, m2y, cbq, (h.y >> 8) & 0xfffu, be, bi);
    score(m2x, m2y, cbq, h.y >> 20, be, bi);
    if (n5 <= (uint32_t)kPfHeadSlots) {
      scored += n5;
      return bi;
    }
    scored += kPfHeadSlots;
  }
  return pf_finish_slow(cur.tail, m2x, m2y, cbq, K, be, bi, &scored);
}

// Polar baseline (paper section 3.5): amplitude |p| to the nearest of the Na
// Lloyd-Max levels (lowest index on ties), phase to the nearest of Np uniform
// bin centres 2 pi i / Np; index = ia * Np + ip.
__device__ __forceinline__ int polar_index(float px, float py, const float* lev, int Na, int Np,
                                           float np_over_2pi) {
  const float r = sqrtf(fmaf(px, px, py * py));
  int ia = 0;
  float bd = INFINITY;
  for (int i = 0; i < Na; ++i) {
    const float d = fabsf(r - lev[i]);
    if (d < bd) {
      bd = d;
      ia = i;
    }
  }
  int ip = (int)floorf(fmaf(atan2f(py, px), np_over_2pi, 0.5f));
  ip = ((ip % Np) + Np) % Np;
  return ia * Np + ip;
}

// Nearest codeword through the prefilter (same result as nearest_all).
__device__ __forceinline__ int nearest_pf(float px, float py, const float4* cbq, int K,
                                          const PrefilterView& pf, unsigned& scored) {
  return pf_finish(pf_locate(px, py, pf), px, py, cbq, K, scored);
}

}  // namespace qamw
