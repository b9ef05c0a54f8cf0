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
//   k_gemm_tc       persistent and warp-specialised.  The work is the sequence
//                   of units (tile of 128 weight rows, group of NT tokens,
//                   K-chunk), chunks fastest; each CTA takes an equal share of
//                   consecutive units.  Eight decode warps gather the codewords
//                   of a chunk and store them (hi, lo) straight into tensor
//                   memory as the A operand (lane = weight row), a copy warp
//                   brings the chunk's B tiles into shared memory, one thread
//                   issues the MMAs into an fp32 accumulator in tensor memory,
//                   and four epilogue warps write the accumulator out as the
//                   partial sum of the CTA's part of the (row tile, token group)
//                   while the next one accumulates in the other buffer.  The
//                   roles meet only at mbarriers (stage ring of A and B tiles,
//                   two accumulator buffers);
//   k_gemm_reduce   Y = bf16(r_i * sum of the partial sums, in CTA order).
#include <algorithm>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

constexpr int kTcRows = 128;  // M of the MMA: weight rows per tile
constexpr int kTcK = 64;      // K-chunk: 64 columns = 32 pairs = one 128-byte row
constexpr int kImgTok = 64;   // tokens per x_bar image
constexpr int kTcDecWarps = 8;          // warps 0-7: decode (two per 32 rows)
constexpr int kTcEpiWarp = 8;           // warps 8-11: epilogue (tensor-memory lane quarters)
constexpr int kTcMmaWarp = 12;          // warp 12: tensor-memory owner, lane 0 issues the MMAs
constexpr int kTcCopyWarp = 13;         // warp 13: lane 0 copies the B tiles
constexpr int kTcThreads = 14 * 32;
constexpr int kTcRepLog2 = 3;           // codeword replicas in the hi/lo table
constexpr int kMinUnits = 4;            // chunks per CTA at least
constexpr int kMaxStages = 4;
constexpr uint32_t kImg = kImgTok * kTcK * 2;    // 8 KB: one binary16 image of 64 tokens
constexpr int kWordStride = 7;  // words per row in a decode warp's word buffer (odd)

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

// Image (c, part, tt) = 8 KB at ((c * 2 + part) * ntt + tt) * 8 KB: row = token
// within the tile of 64, 64 binary16 values of x_bar at columns 64c .. 64c + 63
// (part 0: high, 1: low parts); the images of consecutive token tiles are
// adjacent, so a group of 128 tokens is one 16 KB operand tile.  Tokens from
// ntok to ntt * 64 are zero.  A CTA takes 32 (token, chunk) items: all threads
// form D x / s into shared memory, then one warp rotates the 32 chunks (lane =
// item, consecutive chunks of one token in consecutive lanes, so the shuffles
// of a block > 64 work).
constexpr int kImgItems = 32;
constexpr int kImgThreads = 256;

__global__ void __launch_bounds__(kImgThreads) k_xbar_images(const __nv_bfloat16* __restrict__ x,
                                                             int ntok, int ntt, int d_in, int block,
                                                             uint64_t seed,
                                                             const __half* __restrict__ s,
                                                             const __half* __restrict__ sigma,
                                                             uint8_t* __restrict__ img,
                                                             int32_t* status) {
  __shared__ float buf[kImgItems][kE + 1];
  const int C = d_in / kE;
  const int npad = ntt * kImgTok;
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
        const int tt = (int)(t / kImgTok), row = (int)(t % kImgTok);
        uint8_t* hi = img + ((size_t)(c * 2) * ntt + tt) * kImg;
        uint8_t* lo = hi + (size_t)ntt * kImg;
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

// Instruction descriptor of kind::f16 for N tokens: binary16 A and B (formats
// 0), fp32 accumulator (bits 4-5 = 1), both K-major, N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
template <int NT>
constexpr uint32_t idesc_f16() {
  return (1u << 4) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
}

// One MMA, D (+)= A B^T, with A in tensor memory (lane = row of A, column =
// two binary16 values along K) and B a K-major shared-memory tile.
template <int NT>
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc_f16<NT>()), "r"(accumulate)
      : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// ------------------------------------------------------------ the GEMM

struct GemmTcArgs {
  const uint8_t* packed;
  const float2* codebook;
  const uint8_t* img;  // x_bar images
  float* partial;      // [slot][ntt * 64][d_out] fp32
  int32_t* status;
  int64_t row_bytes;
  int64_t U;  // units: row tiles x token groups x chunks
  int d_out, C, K, ntt, TG, stages;
};

// The CTA (of G) whose share of the U units holds unit v: CTA b holds
// [floor(b U / G), floor((b + 1) U / G)).
__host__ __device__ inline int cta_of(int64_t v, int64_t U, int G) {
  return (int)(((v + 1) * G - 1) / U);
}

// Position in the unit sequence (chunk c of token group tg of row tile rt),
// advanced without divisions.
struct UnitCursor {
  int c, tg, rt;
  __device__ __forceinline__ void start(int64_t v, int C, int TG) {
    const int64_t item = v / C;
    c = (int)(v - item * C);
    rt = (int)(item / TG);
    tg = (int)(item - (int64_t)rt * TG);
  }
  __device__ __forceinline__ void next(int C, int TG) {
    if (++c == C) {
      c = 0;
      if (++tg == TG) {
        tg = 0;
        ++rt;
      }
    }
  }
};

template <int NT>
constexpr uint32_t stage_bytes() {
  return 2 * (uint32_t)NT * 128u;  // B hi, B lo
}

// Tensor memory (all 512 columns): accumulators [2][NT] from column 0, then
// the A tiles of stage s at column 2 NT + 64 s (32 columns of binary16 pairs
// for the high parts, 32 for the low parts; lane = weight row).
constexpr uint32_t kTmemCols = 512;
constexpr int kAStageCols = 64;

// Shared memory: B stages [S][B hi | B lo] (1024-byte aligned) | table uint2
// [K][4] | decode warps' word buffers | bars: A full [S], B full [S], MMA
// done [S], accumulator full [2], accumulator empty [2], final |
// tensor-memory address.  At least 116 KB, so that one CTA (the owner of the
// whole tensor memory) runs per SM.
size_t gemm_tc_smem(uint32_t stage, int S, int K) {
  const size_t need = 1024 + (size_t)S * stage + ((size_t)K << (kTcRepLog2 + 3)) +
                      (size_t)kTcDecWarps * 32 * kWordStride * 4 + (size_t)(3 * S + 5) * 8 + 16;
  return std::max(need, (size_t)116 * 1024);
}

template <int NT>
int gemm_tc_stages(int K) {
  const size_t limit = 227 * 1024;
  int S = std::min(kMaxStages, (int)(kTmemCols - 2 * NT) / kAStageCols);
  while (S > 2 && gemm_tc_smem(stage_bytes<NT>(), S, K) > limit) --S;
  return S;
}

// Words [F, F + NW) of a row's chunk hold the indices of half H (pairs 16 H ..
// 16 H + 15).
template <int BITS, int H>
struct HalfWords {
  static constexpr int F = (16 * H * BITS) >> 5;
  static constexpr int L = (16 * (H + 1) * BITS - 1) >> 5;
  static constexpr int NW = L - F + 1;
};

// Decode warps: warp w decodes half H = w / 4 (pairs 16 H .. 16 H + 15) of the
// 32 rows 32 (w % 4) .. + 31 of every unit into the unit's A stage in tensor
// memory (the warp's lane quarter: lane = row).
// The packed words are loaded coalesced (lane i of load j takes word j * 32 + i
// of the 32 rows' half-chunks), two units ahead, and pass through the warp's
// word buffer to the lane of their row.
template <int BITS, int NT, int H>
__device__ __forceinline__ void decode_role(const GemmTcArgs& a, uint32_t tmem, uint32_t tab_s,
                                            uint32_t* wbuf, uint64_t* afull,
                                            uint64_t* mdone, int64_t v_lo, int64_t v_hi,
                                            int& flags) {
  using HW = HalfWords<BITS, H>;
  constexpr int NW = HW::NW;
  const int lane = threadIdx.x & 31, q4 = (threadIdx.x >> 5) & 3;
  const uint32_t rep8 = (uint32_t)(lane & ((1 << kTcRepLog2) - 1)) << 3;
  // load j of this lane: row rr[j] of the 32, word HW::F + wj[j] of its half
  uint32_t goff[NW], soff[NW];
  int rr[NW];
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    const int f = 32 * j + lane, row = f / NW, wj = f - row * NW;
    rr[j] = row;
    goff[j] = (uint32_t)(row * a.row_bytes) + 4u * (uint32_t)(HW::F + wj);
    soff[j] = (uint32_t)(row * kWordStride + wj);
  }
  auto gload = [&](const UnitCursor& cu, uint32_t (&g)[NW]) {
    const int64_t row0 = (int64_t)cu.rt * kTcRows + 32 * q4;
    const uint8_t* base = a.packed + row0 * a.row_bytes + (size_t)cu.c * BITS * 4;
#pragma unroll
    for (int j = 0; j < NW; ++j)
      g[j] = (row0 + rr[j] < a.d_out) ? __ldg(reinterpret_cast<const uint32_t*>(base + goff[j])) : 0u;
  };
  int s = 0;
  uint32_t u = 0;
  bool ok = true;
  // pf: the unit whose words are loaded next (two ahead of the one decoded)
  UnitCursor pf;
  pf.start(v_lo, a.C, a.TG);
  auto step = [&](int64_t v, uint32_t (&g)[NW]) {
    // this unit's words to the lanes of their rows; unit v + 2's words into g
#pragma unroll
    for (int j = 0; j < NW; ++j) wbuf[soff[j]] = g[j];
    __syncwarp();
    uint32_t w[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) w[j] = wbuf[lane * kWordStride + j];
    __syncwarp();
    if (v + 2 < v_hi) gload(pf, g);
    pf.next(a.C, a.TG);
    // rows past d_out decode index 0: their accumulator rows are never read
    uint2 cw[kQ / 2];
#pragma unroll
    for (int q = 0; q < kQ / 2; ++q) {
      const int bit = (16 * H + q) * BITS - 32 * HW::F, wi = bit >> 5, sh = bit & 31;
      uint32_t id;
      if (sh + BITS <= 32)
        id = w[wi] >> sh;
      else
        id = __funnelshift_r(w[wi], w[wi + 1], sh);
      id &= (1u << BITS) - 1u;
      cw[q] = lds_u2_tc(tab_s + ((id << (kTcRepLog2 + 3)) | rep8));
    }
    // the stage is free once the MMAs of its previous unit are done (a
    // warp-uniform decision: the tensor-memory stores below are warp-wide)
    const bool free_ok = u == 0 || mbar_wait_bounded(&mdone[s], (u - 1) & 1u);
    if (__any_sync(0xffffffffu, !free_ok)) {
      flags |= QAMW_STATUS_TIMEOUT;
      ok = false;
      return;
    }
    // row r = lane 32 q4 + lane of tensor memory; pair 16 H + q -> column
    // 16 H + q of the stage's high (then low) block
    const uint32_t ta = tmem + ((uint32_t)(32 * q4) << 16) +
                        (uint32_t)(2 * NT + kAStageCols * s + 16 * H);
    uint32_t hv[16], lv[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      hv[q] = cw[q].x;
      lv[q] = cw[q].y;
    }
    tc_st16(ta, hv);
    tc_st16(ta + kAStageCols / 2, lv);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    tc_fence_before();
    mbar_arrive(&afull[s]);
    if (++s == a.stages) {
      s = 0;
      ++u;
    }
  };
  uint32_t gA[NW], gB[NW];
  if (v_lo < v_hi) gload(pf, gA);
  pf.next(a.C, a.TG);
  if (v_lo + 1 < v_hi) gload(pf, gB);
  pf.next(a.C, a.TG);
  for (int64_t v = v_lo; v < v_hi && ok; v += 2) {
    step(v, gA);
    if (ok && v + 1 < v_hi) step(v + 1, gB);
  }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kTcThreads, 1) k_gemm_tc(const GemmTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr uint32_t stage = stage_bytes<NT>();
  const int S = a.stages;
  uint2* tab = reinterpret_cast<uint2*>(smem + (size_t)S * stage);
  uint32_t* words = reinterpret_cast<uint32_t*>(tab + ((size_t)a.K << kTcRepLog2));
  uint64_t* afull = reinterpret_cast<uint64_t*>(words + kTcDecWarps * 32 * kWordStride);
  uint64_t* bfull = afull + S;
  uint64_t* mdone = bfull + S;
  uint64_t* accfull = mdone + S;
  uint64_t* accempty = accfull + 2;
  uint64_t* fin = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int64_t v_lo = (int64_t)blockIdx.x * a.U / G;
  const int64_t v_hi = ((int64_t)blockIdx.x + 1) * a.U / G;

  // the hi/lo codeword table needs nothing from the kernels ahead
  for (int j = tid; j < a.K; j += kTcThreads) {
    const float2 c = __ldg(a.codebook + j);
    const uint2 u = split_h2(c.x, c.y);
#pragma unroll
    for (int r = 0; r < (1 << kTcRepLog2); ++r)
      tab[(j << kTcRepLog2) + ((r + lane) & ((1 << kTcRepLog2) - 1))] = u;
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&afull[s], kTcDecWarps * 32);
      mbar_init(&bfull[s], 1);
      mbar_init(&mdone[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 128);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) {  // the accumulators and the A stages
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
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
  int flags = 0;

  if (warp < kTcDecWarps) {
    uint32_t* wbuf = words + warp * 32 * kWordStride;
    if (warp < 4)
      decode_role<BITS, NT, 0>(a, tmem, smem_u32(tab), wbuf, afull, mdone, v_lo, v_hi, flags);
    else
      decode_role<BITS, NT, 1>(a, tmem, smem_u32(tab), wbuf, afull, mdone, v_lo, v_hi, flags);
  } else if (warp < kTcEpiWarp + 4) {
    // epilogue: warp q4 reads lanes (rows) 32 q4 .. + 31 of the accumulator
    const int q4 = warp & 3;
    int n = 0;
    for (int64_t v = v_lo; v < v_hi; ++n) {
      const int64_t item = v / a.C;
      const int64_t v_end = min(v_hi, (item + 1) * a.C);
      const int b = n & 1;
      const bool ok = mbar_wait_bounded(&accfull[b], (uint32_t)(n >> 1) & 1u);
      if (__any_sync(0xffffffffu, !ok)) {
        flags |= QAMW_STATUS_TIMEOUT;
        break;
      }
      tc_fence_after();
      const int rt = (int)(item / a.TG), tg = (int)(item - (int64_t)rt * a.TG);
      const int slot = (int)blockIdx.x - cta_of(item * a.C, a.U, G);
      const int64_t orow = (int64_t)rt * kTcRows + 32 * q4 + lane;
      float* dst = a.partial + ((size_t)slot * a.ntt * kImgTok + (size_t)tg * NT) * a.d_out;
#pragma unroll
      for (int q = 0; q < NT / 16; ++q) {
        float val[16];
        tc_ld16(tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(b * NT + 16 * q), val);
        if (orow < a.d_out) {
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[(size_t)(16 * q + e) * a.d_out + orow] = val[e];
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[b]);
      v = v_end;
    }
  } else if (warp == kTcMmaWarp) {
    if (lane == 0) {
      int s = 0;
      uint32_t u = 0;
      int n = 0;
      bool ok = true;
      for (int64_t v = v_lo; v < v_hi && ok; ++n) {
        const int64_t v_end = min(v_hi, (v / a.C + 1) * a.C);
        const int b = n & 1;
        // the buffer's previous accumulation has been read out
        if (n >= 2 && !mbar_wait_bounded(&accempty[b], (uint32_t)((n >> 1) - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * NT);
        for (bool first = true; v < v_end; ++v, first = false) {
          if (!mbar_wait_bounded(&afull[s], u & 1u) || !mbar_wait_bounded(&bfull[s], u & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bhi = smem_u32(smem + (size_t)s * stage), blo = bhi + NT * 128;
          const uint32_t ahi = tmem + (uint32_t)(2 * NT + kAStageCols * s), alo = ahi + kAStageCols / 2;
#pragma unroll
          for (int k = 0; k < kTcK / 16; ++k) {  // 16 K-columns per MMA: 8 tensor-memory
                                                 // columns of A, 32 bytes of a B row
            const uint64_t dbh = smem_desc_sw128(bhi + 32u * k), dbl = smem_desc_sw128(blo + 32u * k);
            tc_mma_ts<NT>(d, ahi + 8u * k, dbh, (first && k == 0) ? 0u : 1u);
            tc_mma_ts<NT>(d, alo + 8u * k, dbh, 1u);
            tc_mma_ts<NT>(d, ahi + 8u * k, dbl, 1u);
          }
          tc_commit(&mdone[s]);  // the stage is free once these MMAs are done
          if (++s == S) {
            s = 0;
            ++u;
          }
        }
        if (ok) tc_commit(&accfull[b]);
      }
      if (!ok) flags |= QAMW_STATUS_TIMEOUT;
      // every MMA is done before the tensor memory is released
      tc_commit(fin);
      if (!mbar_wait_bounded(fin, 0)) flags |= QAMW_STATUS_TIMEOUT;
    }
  } else if (warp == kTcCopyWarp) {
    if (lane == 0) {
      int s = 0;
      uint32_t u = 0;
      int64_t issued = 0;
      UnitCursor cu;
      cu.start(v_lo, a.C, a.TG);
      for (int64_t v = v_lo; v < v_hi; ++v, cu.next(a.C, a.TG)) {
        if (u > 0 && !mbar_wait_bounded(&mdone[s], (u - 1) & 1u)) {
          flags |= QAMW_STATUS_TIMEOUT;
          break;
        }
        unsigned char* st = smem + (size_t)s * stage;
        const uint8_t* src =
            a.img + ((size_t)(cu.c * 2) * a.ntt + (size_t)cu.tg * (NT / kImgTok)) * kImg;
        mbar_expect_tx(&bfull[s], 2u * NT * 128u);
        bulk_g2s(st, src, NT * 128u, &bfull[s]);
        bulk_g2s(st + NT * 128, src + (size_t)a.ntt * kImg, NT * 128u, &bfull[s]);
        ++issued;
        if (++s == S) {
          s = 0;
          ++u;
        }
      }
      // no copy in flight at exit: the last use of each stage has landed
      for (int64_t j = max((int64_t)0, issued - S); j < issued; ++j)
        if (!mbar_wait_bounded(&bfull[j % S], (uint32_t)(j / S) & 1u)) flags |= QAMW_STATUS_TIMEOUT;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
  raise_flag(a.status, flags);
}

// Y[t][i] = bf16(r_i * sum of the partial sums of (row tile, token group) in
// CTA order).  Block (rt, j): rows 128 rt .. + 127 (one per thread) and tokens
// 8 j .. 8 j + 7, all in one token group (whose partial sums exist for all its
// tokens, padding included).
constexpr int kRedTok = 8;
__global__ void __launch_bounds__(kTcRows) k_gemm_reduce(const float* __restrict__ partial,
                                                         int64_t U, int G, int C, int TG, int NT,
                                                         int ntok_pad, int ntok, int d_out,
                                                         const __half* __restrict__ rnorm,
                                                         __nv_bfloat16* __restrict__ y) {
  const int rt = blockIdx.x, t0 = blockIdx.y * kRedTok;
  const int64_t i = (int64_t)rt * kTcRows + threadIdx.x;
  const int64_t item = (int64_t)rt * TG + t0 / NT;
  const int nseg = cta_of(item * C + C - 1, U, G) - cta_of(item * C, U, G) + 1;
  pdl_wait();
  pdl_trigger();
  if (i >= d_out) return;
  float acc[kRedTok];
#pragma unroll
  for (int j = 0; j < kRedTok; ++j) acc[j] = 0.f;
  for (int s = 0; s < nseg; ++s) {
    const float* src = partial + ((size_t)s * ntok_pad + t0) * d_out + i;
#pragma unroll
    for (int j = 0; j < kRedTok; ++j) acc[j] += __ldg(src + (size_t)j * d_out);
  }
  const float rn = __half2float(rnorm[i]);
#pragma unroll
  for (int j = 0; j < kRedTok; ++j)
    if (t0 + j < ntok) y[(size_t)(t0 + j) * d_out + i] = __float2bfloat16_rn(acc[j] * rn);
}

// The launch plan of a (d_out, d_in, ntok) product on the current device.
struct GemmPlan {
  int NT;      // tokens per tile: 64 or 128
  int TG;      // token groups
  int ntt;     // 64-token images (TG * NT / 64)
  int G;       // CTAs
  int segmax;  // partial sums per (row tile, token group) at most
  int64_t U;   // units
};

GemmPlan plan_gemm(int d_out, int d_in, int ntok) {
  GemmPlan p;
  const int C = d_in / kE;
  p.NT = ntok > kImgTok ? 128 : 64;
  p.TG = (ntok + p.NT - 1) / p.NT;
  p.ntt = p.TG * (p.NT / kImgTok);
  p.U = (int64_t)((d_out + kTcRows - 1) / kTcRows) * p.TG * C;
  p.G = (int)std::min<int64_t>(sm_count(), std::max<int64_t>(1, p.U / kMinUnits));
  // an item of C units meets at most ceil((C - 1) / per) + 1 CTA shares
  const int64_t per = std::max<int64_t>(1, p.U / p.G);
  p.segmax = (int)std::min<int64_t>(p.G, (C - 1 + per - 1) / per + 1);
  return p;
}

template <int BITS, int NT>
cudaError_t run_gemm_tc(const qamw_matrix& m, const uint8_t* img, const GemmPlan& p, float* partial,
                        int32_t* d_status, cudaStream_t stream) {
  GemmTcArgs a;
  a.packed = m.packed;
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.img = img;
  a.partial = partial;
  a.status = d_status;
  a.row_bytes = m.row_bytes;
  a.U = p.U;
  a.d_out = m.d_out;
  a.C = m.d_in / kE;
  a.K = 1 << m.bits;
  a.ntt = p.ntt;
  a.TG = p.TG;
  a.stages = gemm_tc_stages<NT>(a.K);
  const size_t smem = gemm_tc_smem(stage_bytes<NT>(), a.stages, a.K);
  const void* fn = reinterpret_cast<const void*>(&k_gemm_tc<BITS, NT>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(k_gemm_tc<BITS, NT>, dim3(p.G), dim3(kTcThreads), smem, stream, a);
}

template <int BITS>
cudaError_t run_gemm_bits(const qamw_matrix& m, const uint8_t* img, const GemmPlan& p,
                          float* partial, int32_t* d_status, cudaStream_t stream) {
  return p.NT == 128 ? run_gemm_tc<BITS, 128>(m, img, p, partial, d_status, stream)
                     : run_gemm_tc<BITS, 64>(m, img, p, partial, d_status, stream);
}

size_t images_bytes(int C, int ntt) { return (size_t)C * 2 * ntt * kImg; }

}  // namespace

size_t gemm_workspace_bytes(int d_out, int d_in, int ntok) {
  const GemmPlan p = plan_gemm(d_out, d_in, ntok);
  return images_bytes(d_in / kE, p.ntt) +
         (size_t)p.segmax * p.ntt * kImgTok * (size_t)d_out * sizeof(float);
}

cudaError_t launch_decode_gemm(const qamw_matrix& m, const uint16_t* d_x, int ntok, uint16_t* d_y,
                               void* d_ws, int32_t* d_status, cudaStream_t stream) {
  const int C = m.d_in / kE;
  const GemmPlan p = plan_gemm(m.d_out, m.d_in, ntok);
  if (p.U == 0) return cudaSuccess;
  uint8_t* img = static_cast<uint8_t*>(d_ws);
  float* partial = reinterpret_cast<float*>(img + images_bytes(C, p.ntt));
  {
    const int64_t V = (int64_t)p.ntt * kImgTok * C;
    const void* fn = reinterpret_cast<const void*>(&k_xbar_images);
    const int grid = persistent_grid(fn, kImgThreads, 0, (V + kImgItems - 1) / kImgItems);
    cudaError_t err = launch_pdl(k_xbar_images, dim3(grid), dim3(kImgThreads), 0, stream,
                                 reinterpret_cast<const __nv_bfloat16*>(d_x), ntok, p.ntt, m.d_in,
                                 m.block, m.mask_seed, reinterpret_cast<const __half*>(m.chan_scale),
                                 reinterpret_cast<const __half*>(m.sigma), img, d_status);
    if (err != cudaSuccess) return err;
  }
  cudaError_t err;
  switch (m.bits) {
    case 1: err = run_gemm_bits<1>(m, img, p, partial, d_status, stream); break;
    case 2: err = run_gemm_bits<2>(m, img, p, partial, d_status, stream); break;
    case 3: err = run_gemm_bits<3>(m, img, p, partial, d_status, stream); break;
    case 4: err = run_gemm_bits<4>(m, img, p, partial, d_status, stream); break;
    case 5: err = run_gemm_bits<5>(m, img, p, partial, d_status, stream); break;
    case 6: err = run_gemm_bits<6>(m, img, p, partial, d_status, stream); break;
    case 7: err = run_gemm_bits<7>(m, img, p, partial, d_status, stream); break;
    case 8: err = run_gemm_bits<8>(m, img, p, partial, d_status, stream); break;
    case 9: err = run_gemm_bits<9>(m, img, p, partial, d_status, stream); break;
    case 10: err = run_gemm_bits<10>(m, img, p, partial, d_status, stream); break;
    case 11: err = run_gemm_bits<11>(m, img, p, partial, d_status, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (err != cudaSuccess) return err;
  const dim3 rgrid((m.d_out + kTcRows - 1) / kTcRows, (ntok + kRedTok - 1) / kRedTok);
  return launch_pdl(k_gemm_reduce, rgrid, dim3(kTcRows), 0, stream, (const float*)partial, p.U,
                    p.G, C, p.TG, p.NT, p.ntt * kImgTok, ntok, m.d_out,
                    reinterpret_cast<const __half*>(m.row_norm),
                    reinterpret_cast<__nv_bfloat16*>(d_y));
}

}  // namespace qamw
