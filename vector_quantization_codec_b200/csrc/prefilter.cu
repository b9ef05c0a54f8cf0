// prefilter.cu -- exact coarse-grid prefilter for the nearest-codeword search
// (paper section 3.6: "map each normalised pair to its Euclidean-nearest
// codebook entry").
//
// The plane [-R, R)^2 is cut into G x G square cells.  For each cell the table
// lists, in ascending index order, every codeword that can be the nearest one
// (as the encoder computes it in fp32) for some point of the cell:
//   1. D2 = min_j max_{q in cell} |q - c_j|^2   (every point of the cell has a
//      codeword at most sqrt(D2) away, so its nearest one is that close);
//   2. keep j with min_{q in cell} |q - c_j|^2 <= D2 + M;
//   3. drop j when another kept codeword k is closer over the whole cell by
//      more than M: |q - c_j|^2 - |q - c_k|^2 is affine in q, so checking the
//      four corners decides it.
// M bounds the fp32 rounding of the encoder's |c|^2 - 2 p.c scores with a wide
// margin, and cells are grown by eps to cover rounding of the cell index, so a
// list search returns exactly what the exhaustive fp32 search would.  Points
// off the grid (|p| >= R) use the list of their angular sector, built by the
// same dominance test over the unbounded sector region.  Lists that exceed
// kPfCap (none for the codebooks trained here) and non-finite points take the
// exhaustive path.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

__global__ void __launch_bounds__(1024) k_pf_header(const float2* __restrict__ cb, int K, int G,
                                                    PrefilterHeader* __restrict__ hdr) {
  __shared__ float red[32];
  float mr = 0.f;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const float2 c = cb[j];
    mr = fmaxf(mr, sqrtf(c.x * c.x + c.y * c.y));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mr;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mr = fmaxf(mr, red[w]);
    // the grid just covers the codebook; points beyond use the sector lists
    const float R = 1.0625f * mr + 0.0625f;
    PrefilterHeader h;
    h.R = R;
    h.inv_h = (float)G / (2.f * R);
    h.h = 2.f * R / (float)G;
    const float Rp = 1.41421356f * R;  // largest |p| on the grid
    h.margin = ldexpf(mr * mr + 2.f * Rp * mr + 1.f, -18);
    h.G = G;
    h.cap = kPfCap;
    h.K = K;
    h.NS = G > 0 ? kPfSectors : 0;
    h.Gi = prefilter_inner(G);
    *hdr = h;
  }
}

constexpr int kBuildWarps = 8;
constexpr int kMaxCand = 256;

// Tail: slot 0 the count (kPfOverflow when the list did not fit), slots 1..m
// the candidates, the rest zero.  Head: four 16-bit slots with 8 x the first
// four candidates (unused ones repeating the first, scored without a branch
// by the encoder), min(m, 4) - 1 in bits 14-15 of slot 0, and the "more in the
// tail" bit in slot 2.  Called by all 32 lanes of a warp.
__device__ void write_list(void* table, size_t nlists, size_t n, bool overflow, int m,
                           const uint16_t* keep) {
  const int lane = threadIdx.x & 31;
  overflow = overflow || m <= 0;
  uint16_t* tail = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(table) +
                                               prefilter_tails_offset(nlists)) +
                   n * kPfSlots;
  tail[lane] = lane == 0 ? (overflow ? (uint16_t)kPfOverflow : (uint16_t)m)
                         : (!overflow && lane - 1 < m ? keep[lane - 1] : (uint16_t)0);
  if (lane == 0) {
    const uint32_t first = overflow ? 0u : keep[0];
    uint32_t slot[kPfHeadSlots];
    for (int t = 0; t < kPfHeadSlots; ++t)
      slot[t] = (((!overflow && t < m) ? (uint32_t)keep[t] : first) << 3) & 0x3fffu;
    slot[0] |= (uint32_t)((overflow ? kPfHeadSlots : min(m, kPfHeadSlots)) - 1) << 14;
    if (overflow || m > kPfHeadSlots) slot[2] |= kPfMoreBit;
    const uint2 h = make_uint2(slot[0] | (slot[1] << 16), slot[2] | (slot[3] << 16));
    *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(table) + prefilter_lists_offset() +
                              n * 8) = h;
  }
}

// Inner grid, one thread per cell: the ascending union of the four child
// lists, or the "more" bit (more than 4 candidates, or an overflowed child).
__global__ void __launch_bounds__(256) k_pf_inner(void* __restrict__ table) {
  const PrefilterHeader hdr = *reinterpret_cast<const PrefilterHeader*>(table);
  const int G = hdr.G, Gi = hdr.Gi;
  const int cell = blockIdx.x * blockDim.x + threadIdx.x;
  if (cell >= Gi * Gi) return;
  const int ix = cell % Gi, iy = cell / Gi;
  const size_t nlists = (size_t)G * G + hdr.NS;
  const uint16_t* tails = reinterpret_cast<const uint16_t*>(
      reinterpret_cast<const uint8_t*>(table) + prefilter_tails_offset(nlists));
  uint32_t u[kPfHeadSlots];
  int m = 0;
  bool more = false;
  for (int d = 0; d < 4 && !more; ++d) {
    const size_t n = (size_t)(2 * iy + (d >> 1)) * G + (2 * ix + (d & 1));
    const uint16_t* t = tails + n * kPfSlots;
    const uint32_t cnt = t[0];
    if (cnt == kPfOverflow || cnt == 0u) {
      more = true;
      break;
    }
    for (uint32_t k = 1; k <= cnt && !more; ++k) {
      const uint32_t v = t[k];
      int pos = 0;
      while (pos < m && u[pos] < v) ++pos;
      if (pos < m && u[pos] == v) continue;
      if (m == kPfHeadSlots) {
        more = true;
        break;
      }
      for (int q = m; q > pos; --q) u[q] = u[q - 1];
      u[pos] = v;
      ++m;
    }
  }
  uint32_t slot[kPfHeadSlots];
  for (int t = 0; t < kPfHeadSlots; ++t) slot[t] = more ? 0u : ((t < m ? u[t] : u[0]) << 3) & 0x3fffu;
  slot[0] |= (uint32_t)((more ? kPfHeadSlots : m) - 1) << 14;
  if (more) slot[2] |= kPfMoreBit;
  uint2* inner = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(table) +
                                          prefilter_inner_offset(nlists));
  inner[cell] = make_uint2(slot[0] | (slot[1] << 16), slot[2] | (slot[3] << 16));
}

// One warp per cell.
__global__ void __launch_bounds__(kBuildWarps * 32) k_pf_build(const float2* __restrict__ cb,
                                                               void* __restrict__ table) {
  __shared__ uint16_t cand[kBuildWarps][kMaxCand];
  __shared__ uint16_t keep[kBuildWarps][kMaxCand];
  const PrefilterHeader hdr = *reinterpret_cast<const PrefilterHeader*>(table);
  const int G = hdr.G, K = hdr.K;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int cell = blockIdx.x * kBuildWarps + wib;
  if (cell >= G * G) return;
  const int gx = cell % G, gy = cell / G;
  const double R = hdr.R, h = hdr.h, M = hdr.margin;
  const double eps = ldexp(R, -16);
  const double x0 = -R + gx * h - eps, x1 = -R + (gx + 1) * h + eps;
  const double y0 = -R + gy * h - eps, y1 = -R + (gy + 1) * h + eps;

  // Passes 1-2 run in fp32 over all K codewords, with slack (relative 2^-12,
  // far above fp32 rounding) that can only add candidates; the pruning of
  // step 3 is exact (fp64).
  const float fx0 = (float)x0, fx1 = (float)x1, fy0 = (float)y0, fy1 = (float)y1;
  // 1. D2 = min_j maxdist^2(cell, c_j)
  float D2 = INFINITY;
  for (int j = lane; j < K; j += 32) {
    const float2 c = cb[j];
    const float dx = fmaxf(fabsf(fx0 - c.x), fabsf(fx1 - c.x));
    const float dy = fmaxf(fabsf(fy0 - c.y), fabsf(fy1 - c.y));
    D2 = fminf(D2, fmaf(dx, dx, dy * dy));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) D2 = fminf(D2, __shfl_xor_sync(0xffffffffu, D2, o));
  const float bound = D2 * (1.0f + 1.0f / 4096) + 2.0f * (float)M;

  // 2. codewords whose distance to the cell can be within D2 (+M), ascending j
  int n = 0;
  bool overflow = false;
  for (int j0 = 0; j0 < K; j0 += 32) {
    const int j = j0 + lane;
    bool ok = false;
    if (j < K) {
      const float2 c = cb[j];
      const float dx = fmaxf(fmaxf(fx0 - c.x, c.x - fx1), 0.f);
      const float dy = fmaxf(fmaxf(fy0 - c.y, c.y - fy1), 0.f);
      ok = fmaf(dx, dx, dy * dy) <= bound;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, ok);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (ok && pos < kMaxCand) cand[wib][pos] = (uint16_t)j;
    n += __popc(bal);
  }
  if (n > kMaxCand) overflow = true;
  __syncwarp();

  // 3. drop candidates dominated over the whole cell by another candidate
  int m = 0;
  if (!overflow) {
    const double qx[4] = {x0, x1, x0, x1}, qy[4] = {y0, y0, y1, y1};
    for (int t0 = 0; t0 < n; t0 += 32) {
      const int t = t0 + lane;
      bool alive = false;
      if (t < n) {
        alive = true;
        const float2 ca = cb[cand[wib][t]];
        for (int u = 0; u < n && alive; ++u) {
          if (u == t) continue;
          const float2 cbk = cb[cand[wib][u]];
          double worst = INFINITY;  // min over corners of d(q,a)^2 - d(q,k)^2
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const double ax = qx[e] - ca.x, ay = qy[e] - ca.y;
            const double kx = qx[e] - cbk.x, ky = qy[e] - cbk.y;
            worst = fmin(worst, (ax * ax + ay * ay) - (kx * kx + ky * ky));
          }
          if (worst > M) alive = false;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, alive);
      const int pos = m + __popc(bal & ((1u << lane) - 1u));
      if (alive) keep[wib][pos] = cand[wib][t];
      m += __popc(bal);
    }
  }
  __syncwarp();
  write_list(table, (size_t)G * G + hdr.NS, (size_t)cell, overflow || m > kPfCap, m, keep[wib]);
}

// Warp-wide argmin_j |q - c_j|^2 (any minimiser will do: it only seeds the
// dominance test below).
__device__ int warp_nearest(const float2* cb, int K, double qx, double qy) {
  const int lane = threadIdx.x & 31;
  double bd = INFINITY;
  int bj = 0;
  for (int j = lane; j < K; j += 32) {
    const float2 c = cb[j];
    const double d = (qx - c.x) * (qx - c.x) + (qy - c.y) * (qy - c.y);
    if (d < bd) {
      bd = d;
      bj = j;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double od = __shfl_xor_sync(0xffffffffu, bd, o);
    const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
    if (od < bd || (od == bd && oj < bj)) {
      bd = od;
      bj = oj;
    }
  }
  return bj;
}

// Off-grid sector s: the points p = r e(theta), theta in the sector's angle
// range (grown by eps), r >= R_in, lie in the region beyond the chord P0-P1
// between the rays e0 and e1: conv{P0, P1} + cone{e0, e1}.  Codeword j is
// dominated by k over that region when the affine gap
// |q - c_j|^2 - |q - c_k|^2 exceeds M at P0 and P1 and grows along e0 and e1
// (slope at least min_slope, which also covers the fp32 rounding of scores of
// very distant points).
struct SectorGeom {
  double p0x, p0y, p1x, p1y, e0x, e0y, e1x, e1y, M, min_slope;
};

// Single-precision form of `dominated` with doubled margins and a relative
// slack on the gaps: it can only answer "dominated" where the exact test would.
__device__ bool dominated_f(const SectorGeom& g, float2 cj, float2 ck) {
  const float dx = ck.x - cj.x, dy = ck.y - cj.y;
  const float ms = 2.0f * (float)g.min_slope;
  if ((float)g.e0x * dx + (float)g.e0y * dy < ms) return false;
  if ((float)g.e1x * dx + (float)g.e1y * dy < ms) return false;
  const float cj2 = cj.x * cj.x + cj.y * cj.y, ck2 = ck.x * ck.x + ck.y * ck.y;
  const float slack = 2.0f * (float)g.M + 1e-4f * (cj2 + ck2 + 1.0f);
  const float f0 = 2.0f * ((float)g.p0x * dx + (float)g.p0y * dy) + cj2 - ck2;
  const float f1 = 2.0f * ((float)g.p1x * dx + (float)g.p1y * dy) + cj2 - ck2;
  return f0 > slack + 1e-4f * fabsf(f0) && f1 > slack + 1e-4f * fabsf(f1);
}

__device__ bool dominated(const SectorGeom& g, float2 cj, float2 ck) {
  const double dx = (double)ck.x - cj.x, dy = (double)ck.y - cj.y;
  if (g.e0x * dx + g.e0y * dy < g.min_slope) return false;
  if (g.e1x * dx + g.e1y * dy < g.min_slope) return false;
  const double cj2 = (double)cj.x * cj.x + (double)cj.y * cj.y;
  const double ck2 = (double)ck.x * ck.x + (double)ck.y * ck.y;
  // |q-c_j|^2 - |q-c_k|^2 = 2 q.(c_k - c_j) + |c_j|^2 - |c_k|^2
  const double f0 = 2.0 * (g.p0x * dx + g.p0y * dy) + cj2 - ck2;
  const double f1 = 2.0 * (g.p1x * dx + g.p1y * dy) + cj2 - ck2;
  return f0 > g.M && f1 > g.M;
}

constexpr int kRefs = 15;

__global__ void __launch_bounds__(kBuildWarps * 32) k_pf_sectors(const float2* __restrict__ cb,
                                                                 void* __restrict__ table) {
  __shared__ uint16_t cand[kBuildWarps][kMaxCand];
  __shared__ uint16_t keep[kBuildWarps][kMaxCand];
  const PrefilterHeader hdr = *reinterpret_cast<const PrefilterHeader*>(table);
  const int G = hdr.G, K = hdr.K, NS = hdr.NS;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int sct = blockIdx.x * kBuildWarps + wib;
  if (sct >= NS) return;
  const size_t n_list = (size_t)G * G + sct;
  const double pi = 3.14159265358979323846, eps = 1e-4;
  const double t0 = -pi + 2.0 * pi * sct / NS - eps, t1 = -pi + 2.0 * pi * (sct + 1) / NS + eps;
  const double Rin = (double)hdr.R * (1.0 - 1.0 / 1024);
  SectorGeom g;
  g.e0x = cos(t0);
  g.e0y = sin(t0);
  g.e1x = cos(t1);
  g.e1y = sin(t1);
  g.p0x = Rin * g.e0x;
  g.p0y = Rin * g.e0y;
  g.p1x = Rin * g.e1x;
  g.p1y = Rin * g.e1y;
  g.M = hdr.margin;
  g.min_slope = ldexp(1.0 + (double)hdr.R, -16);

  // reference codewords: nearest ones at several radii along e0, e1 and the middle
  int refs[kRefs];
  const double tm = 0.5 * (t0 + t1);
  const double dirs[3][2] = {{g.e0x, g.e0y}, {g.e1x, g.e1y}, {cos(tm), sin(tm)}};
  const double radii[5] = {1.0, 2.0, 4.0, 16.0, 256.0};
  for (int d = 0; d < 3; ++d)
    for (int r = 0; r < 5; ++r)
      refs[d * 5 + r] = warp_nearest(cb, K, Rin * radii[r] * dirs[d][0], Rin * radii[r] * dirs[d][1]);

  // 1. codewords not dominated by any reference, ascending j
  int n = 0;
  for (int j0 = 0; j0 < K; j0 += 32) {
    const int j = j0 + lane;
    bool ok = j < K;
    if (ok) {
      const float2 cj = cb[j];
      for (int r = 0; r < kRefs && ok; ++r)
        if (refs[r] != j && dominated_f(g, cj, cb[refs[r]])) ok = false;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, ok);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (ok && pos < kMaxCand) cand[wib][pos] = (uint16_t)j;
    n += __popc(bal);
  }
  __syncwarp();
  if (n > kMaxCand) {
    write_list(table, (size_t)G * G + NS, n_list, true, 0, keep[wib]);
    return;
  }
  // 2. candidates not dominated by another candidate
  int m = 0;
  for (int u0 = 0; u0 < n; u0 += 32) {
    const int u = u0 + lane;
    bool alive = u < n;
    if (alive) {
      const float2 cj = cb[cand[wib][u]];
      for (int v = 0; v < n && alive; ++v)
        if (v != u && dominated(g, cj, cb[cand[wib][v]])) alive = false;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, alive);
    const int pos = m + __popc(bal & ((1u << lane) - 1u));
    if (alive) keep[wib][pos] = cand[wib][u];
    m += __popc(bal);
  }
  __syncwarp();
  write_list(table, (size_t)G * G + NS, n_list, m > kPfCap, m, keep[wib]);
}

}  // namespace

cudaError_t launch_build_prefilter(const float* d_codebook, int bits, int G, void* d_table,
                                   cudaStream_t stream) {
  const int K = 1 << bits;
  const float2* cb = reinterpret_cast<const float2*>(d_codebook);
  PrefilterHeader* hdr = reinterpret_cast<PrefilterHeader*>(d_table);
  k_pf_header<<<1, 1024, 0, stream>>>(cb, K, G, hdr);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || G == 0) return err;
  const int cells = G * G;
  k_pf_build<<<(cells + kBuildWarps - 1) / kBuildWarps, kBuildWarps * 32, 0, stream>>>(cb, d_table);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int NS = prefilter_sectors(G);
  k_pf_sectors<<<(NS + kBuildWarps - 1) / kBuildWarps, kBuildWarps * 32, 0, stream>>>(cb, d_table);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int Gi = prefilter_inner(G);
  if (Gi > 0) k_pf_inner<<<(Gi * Gi + 255) / 256, 256, 0, stream>>>(d_table);
  return cudaGetLastError();
}

}  // namespace qamw
