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

// Sylvester Hadamard butterflies of span < nb over the N values a thread holds
// (N and nb powers of two).  With nb >= N this is v <- H_N v in natural order;
// with nb < N it is H_nb on each group of nb consecutive values.
template <int N>
__device__ __forceinline__ void fwht_reg(float (&v)[N], int nb) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
    if (h < nb) {
#pragma unroll
      for (int i = 0; i < N; i += 2 * h) {
#pragma unroll
        for (int j = i; j < i + h; ++j) {
          const float a = v[j], b = v[j + h];
          v[j] = a + b;
          v[j + h] = a - b;
        }
      }
    }
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
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
  int32_t pad;
};

constexpr int kPfCap = 32;        // candidates per cell
constexpr uint8_t kPfOverflow = 255;  // count value of a cell searched exhaustively

__host__ __device__ inline int prefilter_grid(int bits) {
  return bits <= 5 ? 0 : (bits <= 7 ? 32 : (bits <= 9 ? 64 : 128));
}

__host__ __device__ inline size_t prefilter_counts_offset() { return sizeof(PrefilterHeader); }

__host__ __device__ inline size_t prefilter_lists_offset(int G) {
  return sizeof(PrefilterHeader) + (((size_t)G * G + 15) / 16) * 16;
}

__host__ __device__ inline size_t prefilter_bytes_for(int bits) {
  const int G = prefilter_grid(bits);
  return prefilter_lists_offset(G) + (size_t)G * G * kPfCap * sizeof(uint16_t);
}

struct PrefilterView {
  float R, inv_h, Gf;
  int G;  // 0: exhaustive search only
  const uint8_t* counts;
  const uint16_t* lists;
};

// A table built for another codebook size is ignored (exhaustive search), so a
// list entry can never index past the K codewords in shared memory.
__device__ __forceinline__ PrefilterView prefilter_view(const void* table, int K) {
  const PrefilterHeader* h = reinterpret_cast<const PrefilterHeader*>(table);
  PrefilterView v;
  v.R = h->R;
  v.inv_h = h->inv_h;
  v.G = (h->K == K && h->cap == kPfCap) ? h->G : 0;
  v.Gf = (float)v.G;
  v.counts = reinterpret_cast<const uint8_t*>(table) + prefilter_counts_offset();
  v.lists = reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(table) +
                                              prefilter_lists_offset(h->G));
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

// Same result as nearest_all: the cell's list holds every codeword that can win
// for a point of the cell, in ascending index order.
__device__ __forceinline__ int nearest_pf(float px, float py, const float4* cbq, int K,
                                          const PrefilterView& pf, unsigned& scored) {
  const float m2x = -2.f * px, m2y = -2.f * py;
  if (pf.G > 0) {
    const float gx = (px + pf.R) * pf.inv_h;
    const float gy = (py + pf.R) * pf.inv_h;
    if (gx >= 0.f && gx < pf.Gf && gy >= 0.f && gy < pf.Gf) {
      const int cell = (int)gy * pf.G + (int)gx;
      const int cnt = __ldg(pf.counts + cell);
      if (cnt != kPfOverflow) {
        scored += (unsigned)cnt;
        const uint16_t* L = pf.lists + (size_t)cell * kPfCap;
        float be = INFINITY;
        int bi = 0;
        for (int t = 0; t < cnt; ++t) {
          const int j = __ldg(L + t);
          const float4 c = cbq[j];
          const float e = fmaf(m2x, c.x, fmaf(m2y, c.y, c.z));
          if (e < be) {
            be = e;
            bi = j;
          }
        }
        return bi;
      }
    }
  }
  return nearest_all(m2x, m2y, cbq, K, scored);
}

}  // namespace qamw
