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
// list search returns exactly what the exhaustive fp32 search would.  Cells
// whose list exceeds kPfCap, and points off the grid, take the exhaustive path.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

__global__ void __launch_bounds__(1024) k_pf_header(const float2* __restrict__ cb, int K, int G,
                                                    PrefilterHeader* __restrict__ hdr) {
  __shared__ float red[2][32];
  float mc = 0.f, mr = 0.f;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const float2 c = cb[j];
    mc = fmaxf(mc, fmaxf(fabsf(c.x), fabsf(c.y)));
    mr = fmaxf(mr, sqrtf(c.x * c.x + c.y * c.y));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
    mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = mc;
    red[1][threadIdx.x >> 5] = mr;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
      mc = fmaxf(mc, red[0][w]);
      mr = fmaxf(mr, red[1][w]);
    }
    const float R = 1.25f * mc + 0.25f;
    PrefilterHeader h;
    h.R = R;
    h.inv_h = (float)G / (2.f * R);
    h.h = 2.f * R / (float)G;
    const float Rp = 1.41421356f * R;  // largest |p| on the grid
    h.margin = ldexpf(mr * mr + 2.f * Rp * mr + 1.f, -18);
    h.G = G;
    h.cap = kPfCap;
    h.K = K;
    h.pad = 0;
    *hdr = h;
  }
}

constexpr int kBuildWarps = 8;
constexpr int kMaxCand = 256;

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
  uint8_t* counts = reinterpret_cast<uint8_t*>(table) + prefilter_counts_offset();
  uint16_t* lists = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(table) +
                                                prefilter_lists_offset(G));
  const int gx = cell % G, gy = cell / G;
  const double R = hdr.R, h = hdr.h, M = hdr.margin;
  const double eps = ldexp(R, -16);
  const double x0 = -R + gx * h - eps, x1 = -R + (gx + 1) * h + eps;
  const double y0 = -R + gy * h - eps, y1 = -R + (gy + 1) * h + eps;

  // 1. D2 = min_j maxdist^2(cell, c_j)
  double D2 = INFINITY;
  for (int j = lane; j < K; j += 32) {
    const float2 c = cb[j];
    const double dx = fmax(fabs(x0 - c.x), fabs(x1 - c.x));
    const double dy = fmax(fabs(y0 - c.y), fabs(y1 - c.y));
    D2 = fmin(D2, dx * dx + dy * dy);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) D2 = fmin(D2, __shfl_xor_sync(0xffffffffu, D2, o));

  // 2. codewords whose distance to the cell can be within D2 (+M), ascending j
  int n = 0;
  bool overflow = false;
  for (int j0 = 0; j0 < K; j0 += 32) {
    const int j = j0 + lane;
    bool ok = false;
    if (j < K) {
      const float2 c = cb[j];
      const double dx = fmax(fmax(x0 - c.x, c.x - x1), 0.0);
      const double dy = fmax(fmax(y0 - c.y, c.y - y1), 0.0);
      ok = dx * dx + dy * dy <= D2 + M;
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
  if (overflow || m > kPfCap) {
    if (lane == 0) counts[cell] = kPfOverflow;
    return;
  }
  uint16_t* L = lists + (size_t)cell * kPfCap;
  for (int t = lane; t < kPfCap; t += 32) L[t] = t < m ? keep[wib][t] : (uint16_t)0;
  if (lane == 0) counts[cell] = (uint8_t)m;
}

}  // namespace

cudaError_t launch_build_prefilter(const float* d_codebook, int bits, void* d_table,
                                   cudaStream_t stream) {
  const int G = prefilter_grid(bits);
  const int K = 1 << bits;
  const float2* cb = reinterpret_cast<const float2*>(d_codebook);
  PrefilterHeader* hdr = reinterpret_cast<PrefilterHeader*>(d_table);
  k_pf_header<<<1, 1024, 0, stream>>>(cb, K, G, hdr);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || G == 0) return err;
  const int cells = G * G;
  k_pf_build<<<(cells + kBuildWarps - 1) / kBuildWarps, kBuildWarps * 32, 0, stream>>>(cb, d_table);
  return cudaGetLastError();
}

}  // namespace qamw
