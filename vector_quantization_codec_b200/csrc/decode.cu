// decode.cu -- QAM-W decoder (paper section 3.2): packed indices -> BF16 rows.
//
// Per pair k of a row: look up codeword c[idx_k], scale by sigma_k and the row
// norm r_hat, apply R_inv = diag(D) blockdiag(H_b) / sqrt(b), divide column j by
// the channel scale s_j, round to BF16.  The kernel is bound by HBM: it reads
// bits/16 bytes and writes 2 bytes per weight.
//
// Work: a row is cut into slices of 32 chunks (2048 columns); one warp decodes
// one (row, slice) tile at a time, lane = chunk, 64 columns per lane.  A CTA
// (12 warps, one per SM) takes a contiguous run of tiles of one (matrix, slice)
// -- a segment -- so the per-column factors its lanes need (sigma of 32 pairs
// in registers, D / (sqrt(b) s) of the slice's 2048 columns in a shared table)
// are set up once per segment, and runs of tiles of many matrices go through
// one launch (qamw_decode_many).
//   - each warp streams its tiles' packed words through its own 2-stage ring of
//     cp.async.bulk copies (mbarrier completion, bounded waits), so warps never
//     wait on one another inside a segment;
//   - codewords come from a shared table of fp32 pairs holding (x + y, x - y)
//     -- the first butterfly stage folded in -- with 8 (K = 2048), 16
//     (K = 1024) or 32 (K <= 512) replicas of every entry, lane l reading
//     replica l mod replicas, so a warp's 32 random lookups rarely collide;
//   - the other butterflies run on float2 registers with packed fp32x2
//     arithmetic (two lanes of work per instruction, rounded as the scalar
//     operations);
//   - the warp's 4 KB output tile is staged in shared memory in the 128-byte
//     swizzled layout (no bank conflicts) and written by one TMA tensor store
//     per tile.
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <type_traits>
#include <utility>
#include <vector>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

constexpr int kDecWarps = 12;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecStages = 2;
constexpr int kSliceChunks = 32;                    // chunks of a slice (one per lane)
constexpr int kSliceCols = kSliceChunks * kE;       // 2048
constexpr size_t kTileBytes = 4096;                 // BF16 output of one tile

// Codeword replicas (log2): 8 for K = 2048, 16 for K = 1024, 32 below, so that
// the table of fp32 pairs takes at most 128 KB.  (A binary16 table would halve
// it, but its rounding alone uses ~70% of the 1e-2 elementwise tolerance on
// columns with small channel scales.)
constexpr int rep_log2(int bits) { return bits >= 11 ? 3 : (bits == 10 ? 4 : 5); }

struct DecodeMat {
  const uint8_t* packed;
  const __half* rnorm;
  const __half* sigma;
  const __half* scale;
  int64_t row_bytes;
  int64_t item0;  // first tile of this matrix in the launch (tiles: slice-major)
  int d_out, d_in, block;
  uint64_t seed;
};

template <int MAXM>
struct DecodeLaunch {
  CUtensorMap out[MAXM];  // BF16 output of matrix i as [d_out][d_in / 64][64]
  DecodeMat m[MAXM];
  const float2* codebook;
  int32_t* status;
  int K;
  int fold;        // table holds (x + y, x - y): every matrix has block >= 2
  int n;           // matrices
  int64_t items;   // tiles in all
};

__host__ __device__ inline int slices_of(int d_in) {
  return (d_in / kE + kSliceChunks - 1) / kSliceChunks;
}

__host__ __device__ inline size_t align1024(size_t v) { return (v + 1023) & ~(size_t)1023; }

// Index Q of a chunk as a byte offset into a table of entries 2^SH bytes apart.
template <int BITS, int Q, int SH>
__device__ __forceinline__ uint32_t extract_off(const uint32_t (&w)[BITS]) {
  constexpr int bit = Q * BITS, wi = bit >> 5, sh = bit & 31;
  constexpr uint32_t mask = ((1u << BITS) - 1u) << SH;
  if constexpr (sh + BITS <= 32) {
    if constexpr (sh >= SH)
      return (w[wi] >> (sh - SH)) & mask;
    else
      return (w[wi] << (SH - sh)) & mask;
  } else {
    return (__funnelshift_r(w[wi], w[wi + 1], sh) << SH) & mask;
  }
}

// v[q] = f_q * (table entry of index q), f_q = sigma_q * r_hat.
template <int BITS, int... Q>
__device__ __forceinline__ void gather2(const uint32_t (&w)[BITS], uint32_t tab_s, uint32_t rep8,
                                        const __half2 (&sg)[16], float rn, float2 (&v)[32],
                                        std::integer_sequence<int, Q...>) {
  constexpr int SH = rep_log2(BITS) + 3;
  (
      [&] {
        const float2 cw = lds_f2(tab_s + (extract_off<BITS, Q, SH>(w) | rep8));
        const float f = ((Q & 1) ? __high2float(sg[Q >> 1]) : __low2float(sg[Q >> 1])) * rn;
        v[Q] = mul2(cw, make_float2(f, f));
      }(),
      ...);
}

constexpr unsigned stage_bytes(int bits) { return 128u * (unsigned)bits; }

// Shared memory (from a 1024-byte aligned base): table float2 [K][replicas]
// (padded to 1 KB) | out tiles [12 warps][4 KB] | rings [12][2][128 bits] |
// gtab float4 [16][32] | bars [12][2] (+ 1 KB of alignment slack).
size_t decode_smem(int K, int bits) {
  return 1024 + align1024((size_t)K << (rep_log2(bits) + 3)) + kDecWarps * kTileBytes +
         (size_t)kDecWarps * kDecStages * stage_bytes(bits) + 16 * 32 * 16 +
         kDecWarps * kDecStages * 8;
}

__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, uint32_t src, int x, int y,
                                               int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Until the bulk stores of this thread have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Until the bulk stores of this thread are complete.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <int BITS, int MAXM>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(const __grid_constant__ DecodeLaunch<MAXM> a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  constexpr int RL = rep_log2(BITS);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the 128-byte swizzle of the output tiles is a function of address bits
  // 4..9: tiles start on 1024-byte boundaries
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const size_t tab_bytes = align1024((size_t)a.K << (RL + 3));
  float2* tab = reinterpret_cast<float2*>(smem);
  uint4* ostage = reinterpret_cast<uint4*>(smem + tab_bytes + warp * kTileBytes);
  unsigned char* rings = smem + tab_bytes + kDecWarps * kTileBytes;
  unsigned char* ring = rings + (size_t)warp * kDecStages * stage_bytes(BITS);
  float4* gtab = reinterpret_cast<float4*>(rings + (size_t)kDecWarps * kDecStages * stage_bytes(BITS));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gtab + 16 * 32) + warp * kDecStages;

  // the codeword table needs nothing from the kernels ahead: replica r of entry
  // j at [j][r], written in a lane-rotated order so that a warp's stores spread
  // over the banks
  for (int j = tid; j < a.K; j += kDecThreads) {
    const float2 c = __ldg(a.codebook + j);
    const float2 t = a.fold ? make_float2(c.x + c.y, c.x - c.y) : c;
#pragma unroll
    for (int r = 0; r < (1 << RL); ++r) tab[(j << RL) + ((r + lane) & ((1 << RL) - 1))] = t;
  }
  if (lane == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // the indices, r_hat, sigma and s come from the kernels ahead
  pdl_wait();
  pdl_trigger();

  const uint32_t tab_s = smem_u32(tab);
  const uint32_t rep8 = (uint32_t)(lane & ((1 << RL) - 1)) << 3;  // this lane's replica
  const uint32_t ostage_s = smem_u32(ostage);
  const int64_t lo = (int64_t)blockIdx.x * a.items / gridDim.x;
  const int64_t hi = ((int64_t)blockIdx.x + 1) * a.items / gridDim.x;
  int mi = 0;
  while (mi + 1 < a.n && a.m[mi + 1].item0 <= lo) ++mi;
  unsigned it = 0;  // this warp's tiles so far (ring position)
  // lane 0: bit s = stage s has had a copy; bit 8 + s = phase parity of its last copy
  unsigned issued = 0;
  int flags = 0;
  bool abort = false;
  for (int64_t i = lo; i < hi;) {
    const DecodeMat& M = a.m[mi];
    const int S = slices_of(M.d_in);
    const int64_t end_m = M.item0 + (int64_t)S * M.d_out;
    if (i >= end_m) {
      ++mi;
      continue;
    }
    const int64_t rel = i - M.item0;
    const int g = (int)(rel / M.d_out);
    const int row_a = (int)(rel - (int64_t)g * M.d_out);
    const int64_t seg_end = min(hi, M.item0 + (int64_t)(g + 1) * M.d_out);
    const int row_b = row_a + (int)(seg_end - i);
    i = seg_end;
    const int C = M.d_in / kE;
    const int nch = min(kSliceChunks, C - g * kSliceChunks);
    const int ntiles = row_b - row_a > warp ? (row_b - row_a - warp + kDecWarps - 1) / kDecWarps : 0;
    const unsigned bytes = (unsigned)((nch * BITS * 4 + 15) & ~15);
    const uint8_t* src0 = M.packed + (int64_t)g * kSliceChunks * BITS * 4;
    const unsigned it0 = it;  // ring position of this segment's first tile
    auto issue = [&](int k) {  // tile k of this warp in this segment
      const unsigned st = (it0 + (unsigned)k) % kDecStages;
      const int row = row_a + warp + k * kDecWarps;
      mbar_expect_tx(&bars[st], bytes);
      bulk_g2s(ring + st * stage_bytes(BITS), src0 + (int64_t)row * M.row_bytes, bytes, &bars[st]);
      // parity of this copy's phase = (number of copies into st so far) & 1
      issued = (issued & (1u << st)) ? (issued ^ (1u << (8 + st))) : (issued | (1u << st));
    };
    if (lane == 0 && !abort)
      for (int k = 0; k < min(kDecStages, ntiles); ++k) issue(k);
    // the slice's output factors g_j = D_j / (sqrt(b) s_j), shared by the CTA
    if (__syncthreads_or(abort)) break;  // every warp is done with the last segment's table
    {
      const float inv_sqrt_b = 1.0f / sqrtf((float)M.block);
      const int col0 = g * kSliceCols;
      for (int t = tid; t < nch * 16; t += kDecThreads) {  // gtab[(j/4)][c] = g of column 64c + j
        const int c = t % nch, j4 = t / nch;
        const int col = col0 + c * kE + 4 * j4;
        const uint2 sv = __ldg(reinterpret_cast<const uint2*>(M.scale + col));
        const float2 lo2 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
        const float2 hi2 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
        const float sv4[4] = {lo2.x, lo2.y, hi2.x, hi2.y};
        float gv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = inv_sqrt_b / sv4[e];
          gv[e] = mask_negative(M.seed, (uint32_t)(col + e)) ? -v : v;
        }
        gtab[j4 * 32 + c] = make_float4(gv[0], gv[1], gv[2], gv[3]);
      }
    }
    // sigma of this lane's 32 pairs (binary16, as stored), into registers
    const bool active = lane < nch;
    __half2 sg[16];
    {
      const uint4* sp = reinterpret_cast<const uint4*>(M.sigma + (int64_t)(g * kSliceChunks + lane) * kQ);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 u = active ? __ldg(sp + t) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) sg[4 * t + e] = *reinterpret_cast<const __half2*>(&uu[e]);
      }
    }
    __syncthreads();
    const int nb = min(M.block, kE);
    const int lanes = max(M.block / kE, 1);
    const CUtensorMap* omap = &a.out[mi];
    // the tiles of this segment; the in-register butterfly stages are
    // straight-line code when the block spans at least a whole chunk (a run-time
    // test per stage would make the compiler move every value back into fixed
    // registers after each stage)
    auto tiles = [&](auto full) {
      constexpr bool FULL = decltype(full)::value;
      for (int k = 0; k < ntiles && !abort; ++k, ++it) {
        const unsigned st = it % kDecStages;
        const int row = row_a + warp + k * kDecWarps;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], (it / kDecStages) & 1u))) {
          flags |= QAMW_STATUS_TIMEOUT;
          abort = true;
          break;
        }
        uint32_t w[BITS];
        {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(ring + st * stage_bytes(BITS)) + lane * BITS;
#pragma unroll
          for (int t = 0; t < BITS; ++t) w[t] = active ? src[t] : 0u;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && k + kDecStages < ntiles) issue(k + kDecStages);
        const float rn = __half2float(M.rnorm[row]);
        float2 v[32];
        gather2<BITS>(w, tab_s, rep8, sg, rn, v, std::make_integer_sequence<int, 32>{});
        // the span-1 stage is in the table
        if constexpr (FULL) {  // block >= 64: every in-register stage, straight-line
          fwht2_stage<1>(v);
          fwht2_stage<2>(v);
          fwht2_stage<4>(v);
          fwht2_stage<8>(v);
          fwht2_stage<16>(v);
        } else {
          fwht2_reg(v, nb);
        }
        fwht2_lanes(v, lanes);
        // the previous tile's store has read its source: the stage can be refilled
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float4 g0 = gtab[(2 * t) * 32 + lane], g1 = gtab[(2 * t + 1) * 32 + lane];
          const float2 p0 = mul2(v[4 * t], make_float2(g0.x, g0.y));
          const float2 p1 = mul2(v[4 * t + 1], make_float2(g0.z, g0.w));
          const float2 p2 = mul2(v[4 * t + 2], make_float2(g1.x, g1.y));
          const float2 p3 = mul2(v[4 * t + 3], make_float2(g1.z, g1.w));
          ostage[lane * 8 + (t ^ (lane & 7))] =
              make_uint4(pack_bf16x2(p0.x, p0.y), pack_bf16x2(p1.x, p1.y), pack_bf16x2(p2.x, p2.y),
                         pack_bf16x2(p3.x, p3.y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        // chunks past the row's end (a ragged last slice) fall outside the
        // tensor and are not written
        if (lane == 0) tma_store_tile(omap, ostage_s, 0, g * kSliceChunks, row);
      }
    };
    if (nb == kE)
      tiles(std::true_type{});
    else
      tiles(std::false_type{});
  }
  // copies still in flight (after a timeout) land before the CTA's shared
  // memory goes away; the output stores complete
  if (lane == 0) {
    for (int s = 0; s < kDecStages; ++s)
      if (issued & (1u << s)) mbar_wait_bounded(&bars[s], (issued >> (8 + s)) & 1u);
    bulk_wait_all();
  }
  raise_flag(a.status, flags);
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// BF16 [d_out][d_in] seen as [d_out][d_in / 64][64] for tile stores of
// {64 columns, 32 chunks, 1 row} in the 128-byte swizzled layout.
bool encode_out_map(CUtensorMap* map, void* out, int d_out, int d_in) {
  const auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kE, (cuuint64_t)(d_in / kE), (cuuint64_t)d_out};
  const cuuint64_t strides[2] = {(cuuint64_t)kE * 2, (cuuint64_t)d_in * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kE, (cuuint32_t)kSliceChunks, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MAXM>
bool fill_launch(DecodeLaunch<MAXM>& L, const qamw_matrix* const* ms, int n, uint16_t* const* outs,
                 int32_t* d_status) {
  L.codebook = reinterpret_cast<const float2*>(ms[0]->codebook);
  L.status = d_status;
  L.K = 1 << ms[0]->bits;
  L.fold = ms[0]->block >= 2;
  L.n = n;
  int64_t item = 0;
  for (int i = 0; i < n; ++i) {
    const qamw_matrix& m = *ms[i];
    DecodeMat& d = L.m[i];
    d.packed = m.packed;
    d.rnorm = reinterpret_cast<const __half*>(m.row_norm);
    d.sigma = reinterpret_cast<const __half*>(m.sigma);
    d.scale = reinterpret_cast<const __half*>(m.chan_scale);
    d.row_bytes = m.row_bytes;
    d.item0 = item;
    d.d_out = m.d_out;
    d.d_in = m.d_in;
    d.block = m.block;
    d.seed = m.mask_seed;
    if (!encode_out_map(&L.out[i], outs[i], m.d_out, m.d_in)) return false;
    item += (int64_t)slices_of(m.d_in) * m.d_out;
  }
  L.items = item;
  return true;
}

template <int BITS, int MAXM>
cudaError_t run_decode(const qamw_matrix* const* ms, int n, uint16_t* const* outs, int32_t* d_status,
                       cudaStream_t stream) {
  static_assert(sizeof(DecodeLaunch<MAXM>) <= 32000, "kernel parameters");
  DecodeLaunch<MAXM> L;
  if (!fill_launch<MAXM>(L, ms, n, outs, d_status)) return cudaErrorInvalidValue;
  if (L.items == 0) return cudaSuccess;
  const size_t smem = decode_smem(L.K, BITS);
  const void* fn = reinterpret_cast<const void*>(&k_decode<BITS, MAXM>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  // one CTA per SM; at least a few tiles per warp
  int64_t grid = (L.items + 4 * kDecWarps - 1) / (4 * kDecWarps);
  grid = std::min<int64_t>(std::max<int64_t>(grid, 1), sm_count());
  return launch_pdl(k_decode<BITS, MAXM>, dim3((unsigned)grid), dim3(kDecThreads), smem, stream, L);
}

constexpr int kManyMax = 64;  // matrices per launch of qamw_decode_many

template <int BITS>
cudaError_t decode_bits(const qamw_matrix* const* ms, int n, uint16_t* const* outs,
                        int32_t* d_status, cudaStream_t stream) {
  if (n == 1) return run_decode<BITS, 1>(ms, 1, outs, d_status, stream);
  for (int i = 0; i < n; i += kManyMax) {
    const cudaError_t err =
        run_decode<BITS, kManyMax>(ms + i, std::min(kManyMax, n - i), outs + i, d_status, stream);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

cudaError_t decode_group(const qamw_matrix* const* ms, int n, uint16_t* const* outs,
                         int32_t* d_status, cudaStream_t stream) {
  switch (ms[0]->bits) {
    case 1: return decode_bits<1>(ms, n, outs, d_status, stream);
    case 2: return decode_bits<2>(ms, n, outs, d_status, stream);
    case 3: return decode_bits<3>(ms, n, outs, d_status, stream);
    case 4: return decode_bits<4>(ms, n, outs, d_status, stream);
    case 5: return decode_bits<5>(ms, n, outs, d_status, stream);
    case 6: return decode_bits<6>(ms, n, outs, d_status, stream);
    case 7: return decode_bits<7>(ms, n, outs, d_status, stream);
    case 8: return decode_bits<8>(ms, n, outs, d_status, stream);
    case 9: return decode_bits<9>(ms, n, outs, d_status, stream);
    case 10: return decode_bits<10>(ms, n, outs, d_status, stream);
    case 11: return decode_bits<11>(ms, n, outs, d_status, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const qamw_matrix& m, uint16_t* d_out, int32_t* d_status,
                          cudaStream_t stream) {
  const qamw_matrix* p = &m;
  return decode_group(&p, 1, &d_out, d_status, stream);
}

cudaError_t launch_decode_many(const qamw_matrix* ms, int n, uint16_t* const* d_outs,
                               int32_t* d_status, cudaStream_t stream) {
  // one launch per run of up to kManyMax matrices with the same table: same
  // bits and codebook, and the first butterfly folded (block >= 2) or not
  std::vector<const qamw_matrix*> group;
  std::vector<uint16_t*> gout;
  auto flush = [&]() -> cudaError_t {
    if (group.empty()) return cudaSuccess;
    const cudaError_t e = decode_group(group.data(), (int)group.size(), gout.data(), d_status, stream);
    group.clear();
    gout.clear();
    return e;
  };
  for (int i = 0; i < n; ++i) {
    if (ms[i].d_out == 0) continue;
    if (!group.empty()) {
      const qamw_matrix& f = *group[0];
      if (f.bits != ms[i].bits || f.codebook != ms[i].codebook || (f.block >= 2) != (ms[i].block >= 2)) {
        const cudaError_t e = flush();
        if (e != cudaSuccess) return e;
      }
    }
    group.push_back(&ms[i]);
    gout.push_back(d_outs[i]);
  }
  return flush();
}

}  // namespace qamw
