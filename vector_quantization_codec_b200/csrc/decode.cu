// decode.cu -- QAM-W decoder (paper section 3.2): packed indices -> BF16 rows.
//
// One thread decodes one chunk of 64 columns (32 pairs) of one row:
//   unpack its 32 indices from `bits` 32-bit words (the chunk's bit range is
//   word aligned: 32 * bits bits), look each codeword up in shared memory,
//   scale pair k by sigma_k, run the inverse Hadamard butterflies (in
//   registers, then across the lanes of the block for b > 64), multiply column
//   j by r_hat * D_j / (sqrt(b) * s_j), round to BF16; the warp then writes its
//   4 KB of output with coalesced 16-byte stores.
// The kernel is bound by HBM: it reads bits/16 bytes and writes 2 bytes per
// weight.
#include <utility>

#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

struct DecodeArgs {
  const uint8_t* packed;
  const __half* rnorm;
  const __half* sigma;
  const __half* scale;
  const float2* codebook;
  __nv_bfloat16* out;
  int32_t* status;
  int64_t row_bytes;
  int d_out, d_in, block, K;
  uint64_t seed;
};

constexpr int kDecThreads = 256;

// x[2q], x[2q+1] = f_q * (table entry of index q), f_q = sigma_q * r_hat; the
// table holds (c.x + c.y, c.x - c.y) when the Hadamard block is at least 2
// (the first butterfly stage, which pairs x[2q] with x[2q + 1]), else c.
template <int BITS, int... Q>
__device__ __forceinline__ void gather_pairs(const uint32_t (&w)[BITS], uint32_t cb_s,
                                             const float4* sg4, int C, float rn, float (&x)[kE],
                                             std::integer_sequence<int, Q...>) {
  (
      [&] {
        const float2 cw = lds_f2(cb_s + extract_off8<BITS, Q>(w));
        const float4 s4 = sg4[(Q / 4) * C];
        const float sq = (Q % 4 == 0) ? s4.x : (Q % 4 == 1) ? s4.y : (Q % 4 == 2) ? s4.z : s4.w;
        const float f = sq * rn;
        x[2 * Q] = cw.x * f;
        x[2 * Q + 1] = cw.y * f;
      }(),
      ...);
}

constexpr int kDecStages = 2;

// Bytes of the input stage of one CTA iteration: its T chunks' words, the row
// padding between them, and 16-byte alignment at both ends.
__host__ __device__ inline unsigned decode_stage_bytes(int threads, int bits) {
  return (unsigned)(((size_t)threads * (bits * 4 + 16) + 32 + 15) & ~(size_t)15);
}

// Position (row, chunk) of a virtual thread v = row C + chunk, advanced by a
// fixed step without a 64-bit division.
struct ChunkPos {
  int64_t r;
  int c;
  __device__ __forceinline__ void advance(int64_t dr, int dc, int C) {
    r += dr;
    c += dc;
    if (c >= C) {
      c -= C;
      ++r;
    }
  }
};

// First byte (16-byte aligned down) and length (16-byte multiple) of the packed
// words of the virtual threads from position p0 to position p1 inclusive.
__device__ __forceinline__ void chunk_span(const DecodeArgs& a, int BITS, const ChunkPos& p0,
                                           const ChunkPos& p1, int64_t& start16,
                                           unsigned& bytes) {
  const int64_t s = p0.r * a.row_bytes + (int64_t)p0.c * BITS * 4;
  const int64_t e = p1.r * a.row_bytes + (int64_t)(p1.c + 1) * BITS * 4;
  start16 = s & ~(int64_t)15;
  bytes = (unsigned)(((e + 15) & ~(int64_t)15) - start16);
}

// Per-column factors live transposed in shared memory, [position in chunk][chunk],
// so that the 32 lanes of a warp (32 consecutive chunks) read 32 consecutive
// words.  The packed words of each grid-stride iteration -- one contiguous byte
// range, since consecutive virtual threads own consecutive chunks -- arrive by
// cp.async.bulk into a 2-stage ring ahead of use (two CTAs fit on an SM).  Each warp's output -- 32
// chunks of 64 BF16 = 4 KB, contiguous in W_hat because virtual thread v owns
// bytes [128 v, 128 v + 128) -- is staged in a swizzled shared tile (16-byte
// unit t of lane l at slot t ^ (l & 7), no bank conflicts on either side) and
// written back with 512-byte coalesced stores.
template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint4* stage = reinterpret_cast<uint4*>(smem);  // [warps][32 lanes][8] output tile
  const unsigned in_bytes = decode_stage_bytes(blockDim.x, BITS);
  unsigned char* in = smem + (size_t)blockDim.x * 128;  // [kDecStages][in_bytes]
  uint64_t* bar = reinterpret_cast<uint64_t*>(in + (size_t)kDecStages * in_bytes);
  int64_t* sstart = reinterpret_cast<int64_t*>(bar + kDecStages);  // first byte of each stage
  int* issued = reinterpret_cast<int*>(sstart + kDecStages);
  float2* cb = reinterpret_cast<float2*>(bar + 2 * kDecStages + 2);
  const int P = a.d_in >> 1, C = a.d_in / kE;
  float4* sg4 = reinterpret_cast<float4*>(cb + a.K);  // [q/4][c]: sigma of pairs 32c + q
  float4* g4 = sg4 + (kQ / 4) * C;                    // [j/4][c]: D/(sqrt(b) s), column 64c + j
  const int64_t V = (int64_t)a.d_out * C;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // grid-stride and in-CTA steps as (rows, chunks)
  const int64_t sdr = stride / C;
  const int sdc = (int)(stride - sdr * C);
  const int bdr = (int)((blockDim.x - 1) / C), bdc = (int)((blockDim.x - 1) % C);
  const ChunkPos last{(int64_t)a.d_out - 1, C - 1};

  // thread 0 issues the stage copies: ipos is the first virtual thread of the
  // next stage to issue
  ChunkPos ipos{0, 0};
  auto issue = [&](int s, int64_t b0) {
    ChunkPos p1 = ipos;
    if (b0 + blockDim.x >= V)
      p1 = last;
    else
      p1.advance(bdr, bdc, C);
    int64_t st16;
    unsigned nb;
    chunk_span(a, BITS, ipos, p1, st16, nb);
    sstart[s] = st16;
    mbar_expect_tx(&bar[s], nb);
    bulk_g2s(in + (size_t)s * in_bytes, a.packed + st16, nb, &bar[s]);
    ++issued[s];
    ipos.advance(sdr, sdc, C);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&bar[s], 1);
      issued[s] = 0;
    }
    fence_mbar_init();
  }
  // table fills: unrolled so that each thread's loads are in flight together;
  // the codewords as (x + y, x - y) when the block is at least 2 (the first
  // butterfly stage, folded into the table)
  const bool fold = a.block >= 2;
#pragma unroll 4
  for (int i = threadIdx.x; i < a.K; i += blockDim.x) {
    const float2 cw = a.codebook[i];
    cb[i] = fold ? make_float2(cw.x + cw.y, cw.x - cw.y) : cw;
  }
  // the indices, r_hat, sigma and s below come from the kernels ahead
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    const int64_t b0 = (int64_t)blockIdx.x * blockDim.x;
    ipos.r = b0 / C;
    ipos.c = (int)(b0 - ipos.r * C);
    for (int s = 0; s < kDecStages; ++s) {
      if (b0 + s * stride >= V) break;
      issue(s, b0 + s * stride);
    }
  }
  fill_quads<kQ>(sg4, a.sigma, P, C, [](int, float v) { return v; });
  const float inv_sqrt_b = 1.0f / sqrtf((float)a.block);
  const uint64_t seed = a.seed;
  fill_quads<kE>(g4, a.scale, a.d_in, C, [=](int j, float sv) {
    const float v = inv_sqrt_b / sv;
    return mask_negative(seed, (uint32_t)j) ? -v : v;
  });
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const uint32_t cb_s = smem_u32(cb);
  uint4* wstage = stage + (threadIdx.x >> 5) * 256;
  const int nb = min(a.block, kE);
  const int lanes = max(a.block / kE, 1);
  uint4* out16 = reinterpret_cast<uint4*>(a.out);
  int flags = 0;
  int it = 0;
  ChunkPos pos;  // this thread's virtual thread
  {
    const int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    pos.r = v0 / C;
    pos.c = (int)(v0 - pos.r * C);
  }
  // r_hat of this thread's row, loaded one iteration ahead
  __half rn_next = (int64_t)blockIdx.x * blockDim.x + threadIdx.x < V ? a.rnorm[pos.r]
                                                                      : __float2half(0.f);
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < V;
       base += stride, ++it, pos.advance(sdr, sdc, C)) {
    const int stg = it % kDecStages;
    const bool active = base + threadIdx.x < V;
    const int64_t row = active ? pos.r : 0;
    const int c = active ? pos.c : 0;
    const float rn = __half2float(rn_next);
    {
      ChunkPos nxt = pos;
      nxt.advance(sdr, sdc, C);
      rn_next = base + stride + threadIdx.x < V ? a.rnorm[nxt.r] : __float2half(0.f);
    }
    const bool ok = mbar_wait_bounded(&bar[stg], (unsigned)(it / kDecStages) & 1u);
    if (__syncthreads_or(!ok)) {
      flags |= QAMW_STATUS_TIMEOUT;
      break;
    }

    uint32_t w[BITS];
    {
      const int64_t off = active ? row * a.row_bytes + (int64_t)c * BITS * 4 - sstart[stg] : 0;
      const uint32_t* src = reinterpret_cast<const uint32_t*>(in + (size_t)stg * in_bytes + off);
#pragma unroll
      for (int t = 0; t < BITS; ++t) w[t] = active ? src[t] : 0u;
    }
    __syncthreads();  // every thread has its words: the stage can be refilled
    if (threadIdx.x == 0) {
      const int64_t b2 = base + (int64_t)kDecStages * stride;
      if (b2 < V) issue(stg, b2);
    }

    float x[kE];
    gather_pairs<BITS>(w, cb_s, sg4 + c, C, rn, x, std::make_integer_sequence<int, kQ>{});
    fwht_reg<kE, 2>(x, nb);  // stage 1 is in the table
    fwht_lanes<kE>(x, lanes);
#pragma unroll
    for (int t = 0; t < kE / 8; ++t) {
      const float4 g0 = g4[(2 * t) * C + c], g1 = g4[(2 * t + 1) * C + c];
      const int j = 8 * t;
      wstage[lane * 8 + (t ^ (lane & 7))] =
          make_uint4(pack_bf16x2(x[j] * g0.x, x[j + 1] * g0.y), pack_bf16x2(x[j + 2] * g0.z, x[j + 3] * g0.w),
                     pack_bf16x2(x[j + 4] * g1.x, x[j + 5] * g1.y), pack_bf16x2(x[j + 6] * g1.z, x[j + 7] * g1.w));
    }
    __syncwarp();
    // unit uu = 32 i + lane of this warp's 4 KB belongs to lane uu / 8, slot uu % 8
    const int64_t wbase = base + (threadIdx.x & ~31);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int uu = 32 * i + lane, owner = uu >> 3, t = uu & 7;
      if (wbase + owner < V) out16[(wbase + owner) * 8 + t] = wstage[owner * 8 + (t ^ (owner & 7))];
    }
    __syncwarp();
  }
  // after a timeout: let the copies still in flight land before this CTA's
  // shared memory goes away
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s)
      if (issued[s] > 0) mbar_wait_bounded(&bar[s], (unsigned)(issued[s] - 1) & 1u);
  }
  raise_flag(a.status, flags);
}

size_t decode_smem(int threads, const DecodeArgs& a, int bits) {
  return (size_t)threads * 128 + (size_t)kDecStages * decode_stage_bytes(threads, bits) +
         (2 * kDecStages + 2) * sizeof(uint64_t) + (size_t)a.K * sizeof(float2) +
         (size_t)(a.d_in / 2) * sizeof(float) + (size_t)a.d_in * sizeof(float);
}

template <int BITS>
cudaError_t run_decode(const DecodeArgs& a, cudaStream_t stream) {
  // 256 threads, or 128 when the per-column tables of a very wide matrix leave
  // no room for a 32 KB staging tile within the 227 KB a CTA may use
  const int threads =
      decode_smem(kDecThreads, a, BITS) <= 227 * 1024 ? kDecThreads : kDecThreads / 2;
  const size_t smem = decode_smem(threads, a, BITS);
  const void* fn = reinterpret_cast<const void*>(&k_decode<BITS>);
  cudaError_t err = allow_smem(fn, smem);
  if (err != cudaSuccess) return err;
  const int64_t V = (int64_t)a.d_out * (a.d_in / kE);
  const int grid = persistent_grid(fn, threads, smem, (V + threads - 1) / threads);
  return launch_pdl(k_decode<BITS>, dim3(grid), dim3(threads), smem, stream, a);
}

}  // namespace

cudaError_t launch_decode(const qamw_matrix& m, uint16_t* d_out, int32_t* d_status,
                          cudaStream_t stream) {
  DecodeArgs a;
  a.status = d_status;
  a.packed = m.packed;
  a.rnorm = reinterpret_cast<const __half*>(m.row_norm);
  a.sigma = reinterpret_cast<const __half*>(m.sigma);
  a.scale = reinterpret_cast<const __half*>(m.chan_scale);
  a.codebook = reinterpret_cast<const float2*>(m.codebook);
  a.out = reinterpret_cast<__nv_bfloat16*>(d_out);
  a.row_bytes = m.row_bytes;
  a.d_out = m.d_out;
  a.d_in = m.d_in;
  a.block = m.block;
  a.K = 1 << m.bits;
  a.seed = m.mask_seed;
  switch (m.bits) {
    case 1: return run_decode<1>(a, stream);
    case 2: return run_decode<2>(a, stream);
    case 3: return run_decode<3>(a, stream);
    case 4: return run_decode<4>(a, stream);
    case 5: return run_decode<5>(a, stream);
    case 6: return run_decode<6>(a, stream);
    case 7: return run_decode<7>(a, stream);
    case 8: return run_decode<8>(a, stream);
    case 9: return run_decode<9>(a, stream);
    case 10: return run_decode<10>(a, stream);
    case 11: return run_decode<11>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qamw
