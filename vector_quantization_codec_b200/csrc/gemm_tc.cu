// gemm_tc.cu -- prefill-size fused decode + GEMM, Y = X W_hat^T for many tokens,
// on the fifth-generation tensor cores (tcgen05, accumulator in tensor memory).
//
// As in the decode-GEMV, W_hat is never formed: with x_bar_t = sigma (.)
// R_fwd(x_t / s) (pair k = coordinates 2k, 2k+1),
//   Y[t][i] = r_i * sum_k < x_bar_t[k], c[idx_ik] >,
// a dense contraction of the gathered codewords (A: weight rows x K) with x_bar
// (B: tokens x K).  Both operands are split into binary16 high and low parts and
// the accumulator takes A_hi B_hi + A_lo B_hi + A_hi B_lo (about 22 significant
// bits; one binary16 operand alone would spend most of the 1e-2 tolerance on
// rows whose output is small).
//
// Kernels:
//   k_xbar_images   x_bar of every token, per K-chunk of 64 columns (32 pairs)
//                   and tile of 64 tokens, as the exact shared-memory image of a
//                   K-major operand tile with the 128-byte swizzle (hi and lo),
//                   so one bulk copy brings a B tile in;
//   k_gemm_tc       a CTA owns 128 weight rows x 64 tokens x a range of K-chunks:
//                   its threads decode the chunk's packed indices into swizzled
//                   A tiles (hi, lo) in shared memory while one thread issues
//                   the MMAs of the chunk before (2-stage ring; completion by
//                   tcgen05.commit on an mbarrier); the fp32 accumulator lives in
//                   64 columns of tensor memory and is written as a partial sum;
//   k_gemm_reduce   Y = bf16(r_i * sum of the K-range partial sums, fixed order).
#include <algorithm>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

constexpr int kTcRows = 128;     // M of the MMA: weight rows per CTA tile
constexpr int kTcTok = 64;       // N of the MMA: tokens per CTA tile
constexpr int kTcK = 64;         // K-chunk: 64 columns = 32 pairs = one 128-byte row
constexpr int kTcThreads = 256;  // two threads per weight row decode a chunk
constexpr int kTcStages = 2;
constexpr int kTcRepLog2 = 2;    // codeword replicas in the hi/lo table
constexpr uint32_t kTileA = kTcRows * kTcK * 2;  // 16 KB: one binary16 A tile
constexpr uint32_t kTileB = kTcTok * kTcK * 2;   // 8 KB: one binary16 B tile
constexpr uint32_t kStage = 2 * kTileA + 2 * kTileB;  // A hi, A lo, B hi, B lo

__host__ __device__ inline int tok_tiles(int ntok) { return (ntok + kTcTok - 1) / kTcTok; }

// binary16 high and low parts of a pair of floats.
__device__ __forceinline__ uint2 split_h2(float a, float b) {
  const __half2 hi = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(hi);
  const __half2 lo = __floats2half2_rn(a - hf.x, b - hf.y);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
}

__device__ __forceinline__ uint2 lds_u2_tc(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Byte offset of 16-byte unit u of row r in a K-major operand tile with the
// 128-byte swizzle (rows of 128 bytes; the tile starts on a 1024-byte boundary).
__host__ __device__ inline uint32_t swz(int r, int u) {
  return (uint32_t)r * 128u + (uint32_t)((u ^ (r & 7)) << 4);
}

// ------------------------------------------------------------ x_bar images

// Image (c, tt, part) = 8 KB at ((c * ntt + tt) * 2 + part) * 8 KB: row = token
// within the tile, 64 binary16 values of x_bar at columns 64c .. 64c + 63.
// A CTA takes 32 (token, chunk) items: all threads form D x / s into shared
// memory, then one warp rotates the 32 chunks (lane = item, consecutive chunks
// of one token in consecutive lanes, so the shuffles of a block > 64 work).
constexpr int kImgItems = 32;
constexpr int kImgThreads = 256;

__global__ void __launch_bounds__(kImgThreads) k_xbar_images(const __nv_bfloat16* __restrict__ x,
                                                             int ntok, int d_in, int block,
                                                             uint64_t seed,
                                                             const __half* __restrict__ s,
                                                             const __half* __restrict__ sigma,
                                                             uint8_t* __restrict__ img,
                                                             int32_t* status) {
  __shared__ float buf[kImgItems][kE + 1];
  const int C = d_in / kE;
  const int ntt = tok_tiles(ntok);
  const int npad = ntt * kTcTok;
  const int64_t V = (int64_t)npad * C;
  const int nb = min(block, kE), lanes = max(block / kE, 1);
  const float inv_sqrt_b = 1.0f / sqrtf((float)block);
  int flags = 0;
  pdl_wait();
  pdl_trigger();
  for (int64_t base = (int64_t)blockIdx.x * kImgItems; base < V;
       base += (int64_t)gridDim.x * kImgItems) {
    for (int e = threadIdx.x; e < kImgItems * kE; e += kImgThreads) {
      const int i = e / kE, j = e - i * kE;
      const int64_t v = base + i;
      float val = 0.f;
      if (v < V) {
        const int64_t t = v / C;
        const int c = (int)(v - t * C);
        if (t < ntok) {
          const int col = c * kE + j;
          const float xv = __bfloat162float(x[t * d_in + col]);
          if (!isfinite(xv)) flags |= QAMW_STATUS_NONFINITE;
          const float q = __fdiv_rn(xv, __half2float(s[col]));
          val = mask_negative(seed, (uint32_t)col) ? -q : q;
        }
      }
      buf[i][j] = val;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
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
        const int tt = (int)(t / kTcTok), row = (int)(t % kTcTok);
        uint8_t* hi = img + ((size_t)(c * ntt + tt) * 2) * kTileB;
        uint8_t* lo = hi + kTileB;
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // unit u: columns 8u .. 8u + 7 = pairs 4u .. 4u + 3
          uint32_t h[4], l[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float f = sg[4 * u + e] * inv_sqrt_b;
            const float a = xv[8 * u + 2 * e] * f, b = xv[8 * u + 2 * e + 1] * f;
            if (fmaxf(fabsf(a), fabsf(b)) > 65504.f) flags |= QAMW_STATUS_RANGE;
            const uint2 p = split_h2(a, b);
            h[e] = p.x;
            l[e] = p.y;
          }
          *reinterpret_cast<uint4*>(hi + swz(row, u)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(lo + swz(row, u)) = make_uint4(l[0], l[1], l[2], l[3]);
        }
      }
    }
    __syncthreads();
  }
  raise_flag(status, flags);
}

// ------------------------------------------------------------ tcgen05 wrappers

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle:
// start address >> 4 (bits 0-13), leading-dimension offset 16 B (bits 16-29,
// unused for this layout), stride between 8-row groups 1024 B (bits 32-45),
// descriptor version 1 (bits 46-47), base offset 0, layout type 2 = 128-byte
// swizzle (bits 61-63).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: binary16 A and B (formats 0), fp32
// accumulator (bits 4-5 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at
// bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kTcTok >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier once every MMA this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct GemmTcArgs {
  const uint8_t* packed;
  const float2* codebook;
  const uint8_t* img;  // x_bar images
  float* partial;      // [splits][ntok pad][d_out] fp32
  int32_t* status;
  int64_t row_bytes;
  int d_out, C, ntok, K, splits, ntt;
};

// Shared memory: stages [2][A hi | A lo | B hi | B lo] (1024-byte aligned) |
// table uint2 [K][4] | bars: B full [2], MMA done [2] | tensor-memory address.
size_t gemm_tc_smem(int K) {
  return 1024 + (size_t)kTcStages * kStage + ((size_t)K << (kTcRepLog2 + 3)) + 4 * 8 + 16;
}

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1) k_gemm_tc(const GemmTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint2* tab = reinterpret_cast<uint2*>(smem + (size_t)kTcStages * kStage);
  uint64_t* bfull = reinterpret_cast<uint64_t*>(tab + ((size_t)a.K << kTcRepLog2));
  uint64_t* mdone = bfull + kTcStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + kTcStages);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // tile: (row tile, token tile, K split), the split fastest
  const int split = blockIdx.x % a.splits;
  const int tt = (blockIdx.x / a.splits) % a.ntt;
  const int rt = blockIdx.x / (a.splits * a.ntt);
  const int c_lo = (int)((int64_t)split * a.C / a.splits);
  const int c_hi = (int)((int64_t)(split + 1) * a.C / a.splits);
  const int nc = c_hi - c_lo;

  // the hi/lo codeword table needs nothing from the kernels ahead
  for (int j = tid; j < a.K; j += kTcThreads) {
    const float2 c = __ldg(a.codebook + j);
    const uint2 u = split_h2(c.x, c.y);
#pragma unroll
    for (int r = 0; r < (1 << kTcRepLog2); ++r)
      tab[(j << kTcRepLog2) + ((r + lane) & ((1 << kTcRepLog2) - 1))] = u;
  }
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&mdone[s], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) {  // 64 columns of tensor memory for the 128 x 64 fp32 accumulator
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTcTok)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the indices and x_bar come from the kernels ahead
  pdl_wait();
  pdl_trigger();

  const int r = tid >> 1, h = tid & 1;  // weight row of the tile, half of the chunk
  const int64_t row = (int64_t)rt * kTcRows + r;
  const bool row_ok = row < a.d_out;
  const uint32_t rep8 = (uint32_t)(lane & ((1 << kTcRepLog2) - 1)) << 3;
  const uint32_t tab_s = smem_u32(tab);
  int flags = 0;
  int issued = 0;  // chunks whose MMAs were committed (to mdone[chunk % 2])
  int done = 0;    // chunks whose commit was waited for
  for (int i = 0; i < nc; ++i) {
    const int c = c_lo + i;
    const int st = i % kTcStages;
    unsigned char* stage = smem + (size_t)st * kStage;
    // the stage is free once the MMAs of chunk i - 2 are done
    if (i >= kTcStages) {
      const int j = i - kTcStages;
      const bool ok = mbar_wait_bounded(&mdone[st], (unsigned)(j / kTcStages) & 1u);
      if (__syncthreads_or(!ok)) {
        flags |= QAMW_STATUS_TIMEOUT;
        break;
      }
      done = j + 1;
    }
    if (tid == 0) {  // B tiles of this chunk and token tile: two 8 KB images
      mbar_expect_tx(&bfull[st], 2 * kTileB);
      bulk_g2s(stage + 2 * kTileA, a.img + ((size_t)(c * a.ntt + tt) * 2) * kTileB, 2 * kTileB,
               &bfull[st]);
    }
    // A tiles: thread (r, h) decodes pairs 16h .. 16h + 15 of the chunk of row r
    // into units 4h .. 4h + 3 of row r (hi and lo)
    {
      uint32_t w[BITS];
      if (row_ok) {
        const uint32_t* src =
            reinterpret_cast<const uint32_t*>(a.packed + row * a.row_bytes) + (size_t)c * BITS;
#pragma unroll
        for (int t = 0; t < BITS; ++t) w[t] = __ldg(src + t);
      } else {
#pragma unroll
        for (int t = 0; t < BITS; ++t) w[t] = 0u;
      }
      uint32_t idx[kQ];
      unpack32<BITS>(w, idx);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t q = h ? idx[16 + 4 * u + e] : idx[4 * u + e];
          uint2 v = lds_u2_tc(tab_s + ((q << (kTcRepLog2 + 3)) | rep8));
          if (!row_ok) v = make_uint2(0u, 0u);
          hi[e] = v.x;
          lo[e] = v.y;
        }
        *reinterpret_cast<uint4*>(stage + swz(r, 4 * h + u)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(stage + kTileA + swz(r, 4 * h + u)) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_proxy_async_smem();  // the A tiles, written by the threads, to the tensor cores
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (!mbar_wait_bounded(&bfull[st], (unsigned)(i / kTcStages) & 1u)) {
        flags |= QAMW_STATUS_TIMEOUT;  // the MMAs of this chunk are skipped
      } else {
        tc_fence_after();
        const uint32_t sa = smem_u32(stage);
        const uint32_t ahi = sa, alo = sa + kTileA, bhi = sa + 2 * kTileA, blo = bhi + kTileB;
#pragma unroll
        for (int k = 0; k < kTcK / 16; ++k) {  // 16 columns (32 bytes) per MMA
          const uint32_t off = 32u * k;
          tc_mma(tmem, smem_desc_sw128(ahi + off), smem_desc_sw128(bhi + off),
                 (i > 0 || k > 0) ? 1u : 0u);
          tc_mma(tmem, smem_desc_sw128(alo + off), smem_desc_sw128(bhi + off), 1u);
          tc_mma(tmem, smem_desc_sw128(ahi + off), smem_desc_sw128(blo + off), 1u);
        }
      }
      tc_commit(&mdone[st]);  // arrives when the MMAs issued so far are done
    }
    issued = i + 1;
  }
  // every committed chunk's MMAs are done before the accumulator is read or the
  // tensor memory released (also after a timeout)
  for (int j = done; j < issued; ++j)
    if (!mbar_wait_bounded(&mdone[j % kTcStages], (unsigned)(j / kTcStages) & 1u))
      flags |= QAMW_STATUS_TIMEOUT;
  tc_fence_after();
  const bool failed = __syncthreads_or(flags & QAMW_STATUS_TIMEOUT);
  // epilogue: warps 0-3 read their 32 lanes (rows) of the accumulator
  if (warp < 4 && nc > 0 && !failed) {
    const int64_t orow = (int64_t)rt * kTcRows + warp * 32 + lane;
    float* dst = a.partial + ((size_t)split * a.ntt * kTcTok + (size_t)tt * kTcTok) * a.d_out;
#pragma unroll
    for (int q = 0; q < kTcTok / 16; ++q) {
      float v[16];
      tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + 16u * q, v);
      if (orow < a.d_out) {
#pragma unroll
        for (int e = 0; e < 16; ++e) dst[(size_t)(16 * q + e) * a.d_out + orow] = v[e];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTok)
                 : "memory");
  }
  raise_flag(a.status, flags);
}

// Y[t][i] = bf16(r_i * sum over splits of partial[split][t][i]), in split order.
__global__ void __launch_bounds__(256) k_gemm_reduce(const float* __restrict__ partial, int splits,
                                                     int ntok_pad, int ntok, int d_out,
                                                     const __half* __restrict__ rnorm,
                                                     __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)ntok * d_out;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / d_out, i = e - t * d_out;
    float sum = 0.f;
    for (int s = 0; s < splits; ++s) sum += partial[((size_t)s * ntok_pad + t) * d_out + i];
    y[e] = __float2bfloat16_rn(sum * __half2float(rnorm[i]));
  }
}

// Splits of the K range: enough CTAs to cover the SMs about twice, at least
// four chunks each.
int gemm_splits(int d_out, int ntok, int C) {
  const int tiles = ((d_out + kTcRows - 1) / kTcRows) * tok_tiles(ntok);
  int s = (2 * sm_count() + tiles - 1) / tiles;
  s = std::min(s, std::max(1, C / 4));
  return std::max(s, 1);
}

template <int BITS>
cudaError_t run_gemm_tc(const qamw_matrix& m, const uint8_t* img, int ntok, float* partial,
                        int splits, int32_t* d_status, cudaStream_t stream) {
  GemmTcArgs a;
  a.packed = m.packed;
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.img = img;
  a.partial = partial;
  a.status = d_status;
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.C = m.d_in / kE;
  a.ntok = ntok;
  a.K = 1 << m.bits;
  a.splits = splits;
  a.ntt = tok_tiles(ntok);
  const size_t smem = gemm_tc_smem(a.K);
  const void* fn = reinterpret_cast<const void*>(&k_gemm_tc<BITS>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int grid = ((m.d_out + kTcRows - 1) / kTcRows) * a.ntt * splits;
  return launch_pdl(k_gemm_tc<BITS>, dim3(grid), dim3(kTcThreads), smem, stream, a);
}

}  // namespace

size_t gemm_workspace_bytes(int d_out, int d_in, int ntok) {
  const int C = d_in / kE;
  const size_t img = (size_t)C * tok_tiles(ntok) * 2 * kTileB;
  const int splits_max = std::max(1, C / 4);
  return img + (size_t)splits_max * tok_tiles(ntok) * kTcTok * (size_t)d_out * sizeof(float);
}

cudaError_t launch_decode_gemm(const qamw_matrix& m, const uint16_t* d_x, int ntok, uint16_t* d_y,
                               void* d_ws, int32_t* d_status, cudaStream_t stream) {
  const int C = m.d_in / kE;
  uint8_t* img = static_cast<uint8_t*>(d_ws);
  float* partial = reinterpret_cast<float*>(img + (size_t)C * tok_tiles(ntok) * 2 * kTileB);
  const int splits = gemm_splits(m.d_out, ntok, C);
  {
    const int64_t V = (int64_t)tok_tiles(ntok) * kTcTok * C;
    const void* fn = reinterpret_cast<const void*>(&k_xbar_images);
    const int grid = persistent_grid(fn, kImgThreads, 0, (V + kImgItems - 1) / kImgItems);
    cudaError_t err = launch_pdl(k_xbar_images, dim3(grid), dim3(kImgThreads), 0, stream,
                                 reinterpret_cast<const __nv_bfloat16*>(d_x), ntok, m.d_in,
                                 m.block, m.mask_seed, reinterpret_cast<const __half*>(m.chan_scale),
                                 reinterpret_cast<const __half*>(m.sigma), img, d_status);
    if (err != cudaSuccess) return err;
  }
  cudaError_t err;
  switch (m.bits) {
    case 1: err = run_gemm_tc<1>(m, img, ntok, partial, splits, d_status, stream); break;
    case 2: err = run_gemm_tc<2>(m, img, ntok, partial, splits, d_status, stream); break;
    case 3: err = run_gemm_tc<3>(m, img, ntok, partial, splits, d_status, stream); break;
    case 4: err = run_gemm_tc<4>(m, img, ntok, partial, splits, d_status, stream); break;
    case 5: err = run_gemm_tc<5>(m, img, ntok, partial, splits, d_status, stream); break;
    case 6: err = run_gemm_tc<6>(m, img, ntok, partial, splits, d_status, stream); break;
    case 7: err = run_gemm_tc<7>(m, img, ntok, partial, splits, d_status, stream); break;
    case 8: err = run_gemm_tc<8>(m, img, ntok, partial, splits, d_status, stream); break;
    case 9: err = run_gemm_tc<9>(m, img, ntok, partial, splits, d_status, stream); break;
    case 10: err = run_gemm_tc<10>(m, img, ntok, partial, splits, d_status, stream); break;
    case 11: err = run_gemm_tc<11>(m, img, ntok, partial, splits, d_status, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (err != cudaSuccess) return err;
  const int64_t n = (int64_t)ntok * m.d_out;
  const void* rfn = reinterpret_cast<const void*>(&k_gemm_reduce);
  const int rgrid = persistent_grid(rfn, 256, 0, (n + 255) / 256);
  return launch_pdl(k_gemm_reduce, dim3(rgrid), dim3(256), 0, stream, (const float*)partial, splits,
                    tok_tiles(ntok) * kTcTok, ntok, m.d_out,
                    reinterpret_cast<const __half*>(m.row_norm), reinterpret_cast<__nv_bfloat16*>(d_y));
}

}  // namespace qamw
