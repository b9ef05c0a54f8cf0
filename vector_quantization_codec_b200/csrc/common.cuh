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
// Quantiser of the row encoder: the joint 2D codebook, the polar baseline
// (section 3.5) or the d = 1 scalar ablation (section 2).
constexpr int kJointMode = 0, kPolarMode = 1, kScalarMode = 2;
constexpr int kQ = 32;  // pairs per thread chunk
// Largest d_in: the encoder keeps 6 bytes per column (D_j s_j and 1/sigma) plus
// a 32 KB codebook in shared memory, within the 227 KB a CTA may use.
constexpr int kMaxDin = 32768;
// Largest token count of the prefill decode-GEMM (qamw_decode_gemm).
constexpr int kMaxTokens = 65536;

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

// Programmatic dependent launch.  The kernels of the encode / decode / GEMV
// path are launched so that each may start while the kernel ahead of it in the
// stream is finishing.  pdl_wait() returns once that kernel has completed and
// its writes are visible (at once when there is no such kernel); every read of
// data another path kernel writes (s, sigma, calibration partials, indices,
// r_hat) and every global write come after it.  Before it a kernel reads only
// data no path kernel writes (W, x, the statistic, the codebook, the search
// table).  pdl_trigger(), called after pdl_wait(), lets the next kernel start:
// when kernel N starts, every kernel before N - 1 has completed.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Packed fp32x2 arithmetic (sm_100): one instruction for two lanes of a
// float2, each rounded exactly like the scalar operation (round to nearest
// even), so a packed butterfly gives bitwise the scalar butterfly's results.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// a - b as fma(b, -1, a): the exact difference rounded once, as a subtraction.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.f, -1.f), a);
}

// Sylvester butterflies of element span 2 H2 .. 32 over 64 values held as 32
// float2 (v[i] = elements 2i, 2i + 1), the stages of span < nb only; the span-1
// stage (within a float2) is the caller's.  Stage order and operand order are
// those of fwht_reg, so the results are bitwise the same.
template <int H2>
__device__ __forceinline__ void fwht2_stage(float2 (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2 * H2) {
#pragma unroll
    for (int j = i; j < i + H2; ++j) {
      const float2 a = v[j], b = v[j + H2];
      v[j] = add2(a, b);
      v[j + H2] = sub2(a, b);
    }
  }
}

__device__ __forceinline__ void fwht2_reg(float2 (&v)[32], int nb) {
  if (2 < nb) fwht2_stage<1>(v);
  if (4 < nb) fwht2_stage<2>(v);
  if (8 < nb) fwht2_stage<4>(v);
  if (16 < nb) fwht2_stage<8>(v);
  if (32 < nb) fwht2_stage<16>(v);
}

// fwht_lanes on float2 registers: the same fma with a +-1 factor per element.
__device__ __forceinline__ void fwht2_lanes(float2 (&v)[32], int lanes) {
  const unsigned lane = threadIdx.x & 31u;
  for (int s = 1; s < lanes; s <<= 1) {
    const float sg = (lane & (unsigned)s) ? -1.f : 1.f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, v[j].x, s);
      o.y = __shfl_xor_sync(0xffffffffu, v[j].y, s);
      v[j] = fma2(sg2, v[j], o);
    }
  }
}

// Generic-proxy accesses to shared memory before this fence are ordered before
// later asynchronous-proxy (bulk copy) accesses of the issuing thread.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
    // lower lane: v + o; upper lane: o - v -- one fma with a +-1 factor, the
    // same single rounding as the add or subtract
    const float sg = (lane & (unsigned)s) ? -1.f : 1.f;
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, v[j], s);
      v[j] = fmaf(sg, v[j], o);
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

// Index Q of a chunk as a byte offset into a table of 8-byte entries
// (8 x index): one shift and one mask (a funnel shift first when the index
// straddles two words).
template <int BITS, int Q>
__device__ __forceinline__ uint32_t extract_off8(const uint32_t (&w)[BITS]) {
  constexpr int bit = Q * BITS, wi = bit >> 5, sh = bit & 31;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << 3;
  if constexpr (sh + BITS <= 32) {
    if constexpr (sh >= 3)
      return (w[wi] >> (sh - 3)) & mask;
    else
      return (w[wi] << (3 - sh)) & mask;
  } else {
    return (__funnelshift_r(w[wi], w[wi + 1], sh) << 3) & mask;
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

// The same table as fill_interleaved in groups of four: element j of chunk c
// (c = j / PERIOD, i = j % PERIOD) at float4 slot (i / 4) * C + c, component
// i % 4, so that one 16-byte shared load gives a thread four consecutive
// entries of its chunk and the 32 lanes of a warp read 512 consecutive bytes.
// Consecutive threads fill consecutive slots.
template <int PERIOD, typename F>
__device__ __forceinline__ void fill_quads(float4* dst, const __half* src, int n, int C, F f) {
  const int slots = n / 4;
#pragma unroll 2
  for (int t = threadIdx.x; t < slots; t += blockDim.x) {
    const int i4 = t / C, c = t - i4 * C;
    const int j = c * PERIOD + i4 * 4;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + j));
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
    dst[t] = make_float4(f(j, lo.x), f(j + 1, lo.y), f(j + 2, hi.x), f(j + 3, hi.y));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------- async bulk copies
// cp.async.bulk global -> shared with mbarrier completion (TMA, no tensor map,
// never multicast).  Every wait is bounded: kSpinLimit polls, each a
// potentially suspending try_wait followed (after the first 64) by a 256 ns
// sleep -- about 8,000 cycles a poll measured on B200, so about a second in all
// -- before the caller gives up.  A copy that lands takes a few polls.
constexpr unsigned kSpinLimit = 1u << 18;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Shared-memory loads at a 32-bit shared address (base + byte offset), so
// that gathers need no 64-bit address arithmetic.  lds_f2_ge loads only when
// n >= k (a predicated load).
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

template <int k>
__device__ __forceinline__ float2 lds_f2_ge(uint32_t n, uint32_t addr) {
  // a defined value for lanes that skip the load: a predicated write to an
  // undefined register would keep that register live back to its first use
  float2 v = make_float2(0.f, 0.f);
  asm volatile(
      "{\n .reg .pred q;\n setp.ge.u32 q, %2, %3;\n @q ld.shared.v2.f32 {%0, %1}, [%4];\n}"
      : "+f"(v.x), "+f"(v.y)
      : "r"(n), "n"(k), "r"(addr));
  return v;
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

// Prefetch [src, src + bytes) into L2 (16-byte aligned, a multiple of 16
// bytes, inside one allocation); no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}" : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity,
                                                  unsigned limit = kSpinLimit) {
  for (unsigned i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i >= 64) __nanosleep(256);  // poll at first: copies usually land within a few tries
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
  int32_t Gi;    // inner grid: G / 2 cells per side, heads only (0: none)
};

// Each cell's (or sector's) list: the count and the candidate indices in
// ascending order.  It is stored twice:
//   head (8 bytes, one per list, all heads side by side): four 16-bit slots,
//     slot k holding 8 x (index of candidate k) -- the candidate's byte offset
//     in a float2 codeword table -- in bits 0-13; slots past the count repeat
//     the first candidate.  Bits 14-15 of slot 0: min(count, 4) - 1.  Bit 14
//     of slot 2: the list has more than 4 candidates (the rest are in the
//     tail) or overflowed.  One 8-byte load and four scores resolve almost
//     every point.
//   tail (64 bytes): 32 uint16 slots, slot 0 the exact count (kPfOverflow:
//     search exhaustively), slots 1..count the candidates.
constexpr int kPfSlots = 32;
constexpr int kPfCap = kPfSlots - 1;         // candidates per list
constexpr uint32_t kPfOverflow = 0xffffu;
constexpr int kPfHeadSlots = 4;
constexpr uint32_t kPfMoreBit = 0x4000u;     // in the upper word of a head

// Cells per side of the encoder's table: about 8 sqrt(K) rounded up to a
// power of two, so that near the origin a cell is under half a Voronoi cell
// across and, for Lloyd codebooks of N(0, I_2), lists longer than 4 are rare
// (K >= 8; smaller codebooks are searched exhaustively).  K = 2048: 512 x 512.
__host__ __device__ inline int prefilter_grid(int bits) {
  return bits < 3 ? 0 : 1 << ((bits + 8) / 2);
}

// The training table is rebuilt every Lloyd iteration: one step coarser.
__host__ __device__ inline int prefilter_grid_train(int bits) {
  return bits <= 5 ? 0 : (bits <= 7 ? 64 : (bits <= 9 ? 128 : 256));
}

__host__ __device__ inline size_t prefilter_lists_offset() {
  return (sizeof(PrefilterHeader) + 15) / 16 * 16;
}

// Points off the grid are looked up by angle in kPfSectors equal sectors of
// the region |p| >= R (list of every codeword that can win there).
constexpr int kPfSectors = 256;

__host__ __device__ inline int prefilter_sectors(int G) { return G > 0 ? kPfSectors : 0; }

// The inner grid has cells twice as wide (G / 2 per side, over the same
// square); cell (ix, iy) covers main cells 2ix..2ix+1 x 2iy..2iy+1 and its head
// holds the union of their lists (ascending), or the "more" bit when that
// union has more than 4 candidates or a child list overflowed.  It exists to
// be copied, in part, into shared memory.
__host__ __device__ inline int prefilter_inner(int G) { return G / 2; }

// Bytes of a table with G x G cells: header, heads, tails, inner heads.
__host__ __device__ inline size_t prefilter_bytes_for(int G) {
  const size_t n = (size_t)G * G + prefilter_sectors(G);
  const size_t gi = (size_t)prefilter_inner(G);
  return prefilter_lists_offset() + ((n * 8 + 15) / 16) * 16 + n * kPfSlots * sizeof(uint16_t) +
         gi * gi * 8;
}

// List n (cells 0..G*G-1, then sectors): head at heads[n] (8 bytes), tail at
// tails[n] (32 uint16).
__host__ __device__ inline size_t prefilter_tails_offset(size_t nlists) {
  return prefilter_lists_offset() + ((nlists * 8 + 15) / 16) * 16;
}

// Inner heads, row-major [Gi][Gi] (16-byte aligned).
__host__ __device__ inline size_t prefilter_inner_offset(size_t nlists) {
  return prefilter_tails_offset(nlists) + nlists * kPfSlots * sizeof(uint16_t);
}

struct PrefilterView {
  float R, inv_h, Gf;
  float Rih;  // R * inv_h: grid coordinate of p = fma(p, inv_h, Rih)
  int G;  // 0: exhaustive search only
  int NS;
  const uint2* heads;     // [G*G + NS]
  const uint16_t* tails;  // [G*G + NS][32]
  const uint2* inner;     // [Gi][Gi]
  int Gi;
};

// A table built for another codebook size is ignored (exhaustive search), so a
// list entry can never index past the K codewords in shared memory.
__device__ __forceinline__ PrefilterView prefilter_view(const void* table, int K) {
  const PrefilterHeader* h = reinterpret_cast<const PrefilterHeader*>(table);
  PrefilterView v;
  v.R = h->R;
  v.inv_h = h->inv_h;
  v.Rih = h->R * h->inv_h;
  v.G = (h->K == K && h->cap == kPfCap && h->NS == kPfSectors) ? h->G : 0;
  v.NS = h->NS;
  v.Gf = (float)v.G;
  const size_t nlists = (size_t)h->G * h->G + h->NS;
  v.heads = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(table) +
                                           prefilter_lists_offset());
  v.tails = reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(table) +
                                              prefilter_tails_offset(nlists));
  v.inner = reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(table) +
                                           prefilter_inner_offset(nlists));
  v.Gi = v.G > 0 ? h->Gi : 0;
  return v;
}

// Codeword j sits in shared memory as a plain (x, y) pair.  The nearest
// codeword of p minimises |c|^2 - 2 p.c (= |p - c|^2 - |p|^2), with |c|^2
// formed as fma(x, x, y * y): three FMAs and a multiply per candidate.
__device__ __forceinline__ float score_cw(float m2x, float m2y, float2 c) {
  return fmaf(m2x, c.x, fmaf(m2y, c.y, fmaf(c.x, c.x, c.y * c.y)));
}

__device__ __forceinline__ void score2(float m2x, float m2y, const float2* cb, uint32_t j,
                                       float& be, int& bi) {
  const float e = score_cw(m2x, m2y, cb[j]);
  if (e < be) {
    be = e;
    bi = (int)j;
  }
}

// Exhaustive search, ascending j with a strict '<' (lowest index on ties).
// `scored` accumulates the number of codewords evaluated.
__device__ __forceinline__ int nearest_all2(float m2x, float m2y, const float2* cb, int K,
                                            unsigned& scored) {
  scored += (unsigned)K;
  float be = INFINITY;
  int bi = 0;
  for (int j = 0; j < K; ++j) score2(m2x, m2y, cb, (uint32_t)j, be, bi);
  return bi;
}

// List number of a point: its cell, or for a point off the grid the angular
// sector; kPfNoList without a table or for a point that is not finite.
constexpr uint32_t kPfNoList = 0xffffffffu;
// Head given to points without a list (never written by the builder, whose
// slots stay below 0x4000): bit 15 of slot 2.
constexpr uint32_t kPfNoListBit = 0x8000u;

__device__ __forceinline__ uint32_t pf_list(float px, float py, const PrefilterView& pf) {
  uint32_t n = kPfNoList;
  if (pf.G > 0) {
    const float gx = fmaf(px, pf.inv_h, pf.Rih);
    const float gy = fmaf(py, pf.inv_h, pf.Rih);
    if (gx >= 0.f && gx < pf.Gf && gy >= 0.f && gy < pf.Gf) {
      n = (uint32_t)((int)gy * pf.G + (int)gx);
    } else if (isfinite(px) && isfinite(py)) {
      const float t = (atan2f(py, px) + 3.14159265f) * ((float)pf.NS * 0.159154943f);
      n = (uint32_t)(pf.G * pf.G + min(max((int)t, 0), pf.NS - 1));
    }
  }
  return n;
}

// The head of a point's list (fetched ahead of its scoring by the callers).
__device__ __forceinline__ uint2 pf_head(float px, float py, const PrefilterView& pf) {
  const uint32_t n = pf_list(px, py, pf);
  return n == kPfNoList ? make_uint2(0u, kPfNoListBit) : __ldg(pf.heads + n);
}

// The four head slots of a list scored against p (m2 = -2 p): slot t is
// loaded only when t < min(count, 4) (a predicated shared load: lanes with
// short lists add no traffic) and otherwise scores +inf; the minimum is taken
// as a tree in which the left operand wins ties (the slots hold ascending
// indices).  Returns the best score and its byte offset.
__device__ __forceinline__ void pf_score_head(uint2 h, float m2x, float m2y, uint32_t base,
                                              float& ea, uint32_t& oa) {
  const uint32_t hx = h.x, hy = h.y;
  const uint32_t o0 = hx & 0x3fffu, o1 = hx >> 16, o2 = hy & 0x3fffu, o3 = hy >> 16;
  const uint32_t n4 = (hx >> 14) & 3u;  // min(count, 4) - 1
  const float e0 = score_cw(m2x, m2y, lds_f2(base + o0));
  const float s1 = score_cw(m2x, m2y, lds_f2_ge<1>(n4, base + o1));
  const float s2 = score_cw(m2x, m2y, lds_f2_ge<2>(n4, base + o2));
  const float s3 = score_cw(m2x, m2y, lds_f2_ge<3>(n4, base + o3));
  const float e1 = n4 >= 1u ? s1 : INFINITY;
  const float e2 = n4 >= 2u ? s2 : INFINITY;
  const float e3 = n4 >= 3u ? s3 : INFINITY;
  float eb = e2;
  uint32_t ob = o2;
  ea = e0;
  oa = o0;
  if (e1 < ea) {
    ea = e1;
    oa = o1;
  }
  if (e3 < eb) {
    eb = e3;
    ob = o3;
  }
  if (eb < ea) {
    ea = eb;
    oa = ob;
  }
}

// Rare ends of pf_finish2, for a head with the "more" or the no-list bit: a
// list longer than the head continues in its tail (the point's list n,
// recomputed) from slot 5 with the best of the head as the incumbent; an
// overflowed list or a point without a list (no table, or not finite) is
// searched exhaustively.
__device__ __forceinline__ int pf_finish_rare(uint2 h, float px, float py, const float2* cb, int K,
                                              const PrefilterView& pf, float be, int bi,
                                              unsigned& scored, bool count) {
  const float m2x = -2.f * px, m2y = -2.f * py;
  const uint32_t head_cnt = ((h.x >> 14) & 3u) + 1u;
  if (h.y & kPfNoListBit) {
    if (count) scored -= head_cnt;
    return nearest_all2(m2x, m2y, cb, K, scored);
  }
  const uint16_t* tail = pf.tails + (size_t)pf_list(px, py, pf) * kPfSlots;
  const uint32_t cnt = __ldg(tail);
  if (cnt == kPfOverflow) {
    if (count) scored -= head_cnt;
    return nearest_all2(m2x, m2y, cb, K, scored);
  }
  if (count) scored += cnt - kPfHeadSlots;
  for (uint32_t t = kPfHeadSlots + 1; t <= cnt; ++t) score2(m2x, m2y, cb, __ldg(tail + t), be, bi);
  return bi;
}

// Nearest codeword of p from its list head; the same index as nearest_all2.
// With `count`, `scored` accumulates the distinct candidates of each list.
__device__ __forceinline__ int pf_finish2(uint2 h, float px, float py, const float2* cb, int K,
                                          const PrefilterView& pf, unsigned& scored, bool count) {
  float ea;
  uint32_t oa;
  pf_score_head(h, -2.f * px, -2.f * py, smem_u32(cb), ea, oa);
  if (count) scored += ((h.x >> 14) & 3u) + 1u;
  if (!(h.y & (kPfMoreBit | kPfNoListBit))) return (int)(oa >> 3);
  return pf_finish_rare(h, px, py, cb, K, pf, ea, (int)(oa >> 3), scored, count);
}

// pf_finish2's common path alone: the index, or kPfRare when the head has the
// "more" or the no-list bit (the caller then runs the full search apart from
// its hot loop).  Counts only what it resolves.
constexpr uint32_t kPfRare = 0xffffffffu;
__device__ __forceinline__ uint32_t pf_finish_fast(uint2 h, float px, float py, uint32_t cb_s,
                                                   unsigned& scored, bool count) {
  float ea;
  uint32_t oa;
  pf_score_head(h, -2.f * px, -2.f * py, cb_s, ea, oa);
  const bool rare = (h.y & (kPfMoreBit | kPfNoListBit)) != 0u;
  if (count && !rare) scored += ((h.x >> 14) & 3u) + 1u;
  return rare ? kPfRare : (oa >> 3);
}

// Head of p's list for a caller holding the inner-grid cells [c0, c0 + S)^2
// in shared memory (hs, row-major S x S): that copy when p falls in it and the
// union there fits the head, else the main table (a predicated global load).
// Without a branch: a point off the grid (or without a table) gets the no-list
// head, which the caller resolves with the full search.  p must be finite
// (the encoder stores rows whose points would not be as zero rows); the grid
// test on floor(g) is then the float test 0 <= g < G of pf_list, with G a power
// of two.
__device__ __forceinline__ uint2 pf_head_shared(float px, float py, const PrefilterView& pf,
                                                const uint2* hs, int S, int c0) {
  const int ix = __float2int_rd(fmaf(px, pf.inv_h, pf.Rih));
  const int iy = __float2int_rd(fmaf(py, pf.inv_h, pf.Rih));
  const bool in_grid = ((unsigned)(ix | iy)) < (unsigned)pf.G;
  const unsigned sx = (unsigned)((ix >> 1) - c0), sy = (unsigned)((iy >> 1) - c0);
  const bool in_sq = in_grid & (sx < (unsigned)S) & (sy < (unsigned)S);
  uint2 h = make_uint2(0u, kPfMoreBit);
  if (in_sq) h = hs[sy * S + sx];
  if (in_grid & ((h.y & kPfMoreBit) != 0u)) h = __ldg(pf.heads + (iy * pf.G + ix));
  return in_grid ? h : make_uint2(0u, kPfNoListBit);
}

__device__ __forceinline__ int nearest_pf2(float px, float py, const float2* cb, int K,
                                           const PrefilterView& pf, unsigned& scored, bool count) {
  return pf_finish2(pf_head(px, py, pf), px, py, cb, K, pf, scored, count);
}

// d = 1 ablation: each coordinate to the nearest of the L levels (ascending,
// strict '<', lowest index on ties); index = ix * L + iy.
__device__ __forceinline__ int scalar_index(float px, float py, const float* lev, int L) {
  int ix = 0, iy = 0;
  float bx = INFINITY, by = INFINITY;
  for (int i = 0; i < L; ++i) {
    const float dx = fabsf(px - lev[i]), dy = fabsf(py - lev[i]);
    if (dx < bx) {
      bx = dx;
      ix = i;
    }
    if (dy < by) {
      by = dy;
      iy = i;
    }
  }
  return ix * L + iy;
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


}  // namespace qamw
