// bl_block.cu - the per-256-block scale variant of the BitLinear.
//
// "Core AI model zoo - BitVLA", section 2 ("Generalizing the ternary kernel"),
// contrasts BitNet's per-row scale D [N, 1] with BitCPM's per-256-block scale
// and defines no more of the latter. Reading taken here: a block is 256
// consecutive columns of one row (the last block of a row holds K % 256
// columns when that is not zero); each block is quantised with the per-tensor
// absmean formula of section 1 applied to the block alone; D is fp32
// [N, ceil(K/256)]; the output is the fp32 sum, in ascending block order, of
// the per-block terms t_b = RN(RN(float(acc_b) / s_x) * D[n, b]).
//
// Kernels:
//   bl_block_scale_pack_kernel     one warp per block: exact block mean of |W| (an fp64
//                         interval, with an exact integer comparison when an
//                         fp32 rounding boundary lies inside it), ternarise,
//                         pack 16 codes per word, D[n, b].
//   bl_block_scale_forward_kernel  CTA = 8 warps over a tile of up to TM tokens and a
//                         range of rows; one warp per row at a time. The
//                         tile's activation codes (private order, from the
//                         ActQuant kernel) and their per-block sums sit in
//                         shared memory. Lanes read 32-bit packed words (rows
//                         need not be 16-byte aligned), contract 4 codes per
//                         dp4a, reduce each 16-word block across a half-warp,
//                         and add the block terms in order with shuffles.
#include "bl_internal.h"

#include <algorithm>

namespace bl {
namespace {

constexpr int kLimbs = 9;  // 288 bits: 256 values below 2^277 units of 2^-149

// Sign of (sum_j |w[j]| - B), exactly, for j < cnt. The sum is formed in units
// of 2^-149 in 32-bit limbs: |w| = m * 2^(max(e,1) - 150) = (m << (max(e,1)-1))
// units. B is an fp64 value that is an integer multiple of 2^-149 (the
// midpoint of two fp32 values times a multiple of 16). One thread; used only
// when the fp64 interval cannot decide the rounding.
__device__ __noinline__ int compare_abs_sum(const float* __restrict__ w, int cnt, double B) {
  uint32_t A[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) A[i] = 0u;
  for (int j = 0; j < cnt; ++j) {
    const uint32_t b = __float_as_uint(__ldg(w + j)) & 0x7FFFFFFFu;
    uint32_t e = b >> 23, m = b & 0x7FFFFFu;
    if (e != 0u) m |= 0x800000u; else e = 1u;
    const int sh = (int)e - 1;  // 0 .. 253
    const int limb = sh >> 5;   // 0 .. 7
    const unsigned long long v = (unsigned long long)m << (sh & 31);
    unsigned long long s = (unsigned long long)A[limb] + (uint32_t)v;
    A[limb] = (uint32_t)s;
    s = (unsigned long long)A[limb + 1] + (uint32_t)(v >> 32) + (s >> 32);
    A[limb + 1] = (uint32_t)s;
    unsigned long long c = s >> 32;
    for (int i = limb + 2; c != 0ull && i < kLimbs; ++i) {
      s = (unsigned long long)A[i] + c;
      A[i] = (uint32_t)s;
      c = s >> 32;
    }
  }
  // B = mant * 2^(e - 1075) = (mant << (e - 926)) units of 2^-149.
  const unsigned long long bb = (unsigned long long)__double_as_longlong(B);
  const int be = (int)((bb >> 52) & 0x7FF);
  unsigned long long mant = (bb & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  int sh = be - 926;
  if (sh < 0) {  // the bits shifted out are zero: B is a multiple of 2^-146
    mant >>= -sh;
    sh = 0;
  }
  uint32_t Bl[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) Bl[i] = 0u;
  const int limb = sh >> 5, bit = sh & 31;
  if (limb < kLimbs) Bl[limb] = (uint32_t)(mant << bit);
  if (limb + 1 < kLimbs) Bl[limb + 1] = (uint32_t)(bit ? (mant >> (32 - bit)) : (mant >> 32));
  if (limb + 2 < kLimbs) Bl[limb + 2] = (uint32_t)(bit ? (mant >> (64 - bit)) : 0ull);
  for (int i = kLimbs - 1; i >= 0; --i) {
    if (A[i] != Bl[i]) return A[i] > Bl[i] ? 1 : -1;
  }
  return 0;
}

// One warp per (row, block). Lane l holds columns 4l..4l+3 and 128+4l..128+4l+3
// of the block; four lanes make one packed word.
__global__ void __launch_bounds__(256) bl_block_scale_pack_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                         uint32_t* __restrict__ packed, float* __restrict__ D,
                                                         uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t nb = (K + kScaleBlock - 1) / kScaleBlock;
  const int64_t total = N * nb;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); blk < total; blk += warps) {
    const int64_t n = blk / nb, b = blk - n * nb;
    const int64_t k0 = b * kScaleBlock;
    const int cnt = (int)std::min<int64_t>(kScaleBlock, K - k0);
    const float* src = W + n * K + k0;
    float4 v[2];
    bool ok[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = 128 * h + 4 * lane;
      ok[h] = c < cnt;
      v[h] = ok[h] ? __ldg(reinterpret_cast<const float4*>(src + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // Non-finite weights: record and leave this block unwritten.
    bool bad = false;
    double s = 0.0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float f[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        bad |= (__float_as_uint(f[i]) & 0x7F800000u) == 0x7F800000u;
        s += (double)fabsf(f[i]);
      }
    }
    if (__any_sync(0xFFFFFFFFu, bad)) {
      if (lane == 0) atomicOr(status, 1u);
      continue;
    }
    // Butterfly sum: every lane ends with the same value (fp64 addition is
    // commutative). Depth 7 + 5 = 12 roundings of non-negative terms, so the
    // exact sum T satisfies |S - T| <= 12 * 2^-53 * T < 2^-48 * S.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    const double lo = __ddiv_rd(__dmul_rd(s, 1.0 - 0x1p-48), (double)cnt);
    const double hi = __ddiv_ru(__dmul_ru(s, 1.0 + 0x1p-48), (double)cnt);
    const float c1 = __double2float_rn(lo), c2 = __double2float_rn(hi);
    float mean = c1;
    if (c1 != c2) {
      // c1 < c2 are neighbours; the exact mean rounds to c1 below their
      // midpoint, to c2 above it, to the even one on it. Midpoint * cnt is
      // exact in fp64 (25 + 9 significant bits).
      int cmp = 0;
      if (lane == 0) cmp = compare_abs_sum(src, cnt, 0.5 * ((double)c1 + (double)c2) * (double)cnt);
      cmp = __shfl_sync(0xFFFFFFFFu, cmp, 0);
      mean = cmp < 0 ? c1 : (cmp > 0 ? c2 : ((__float_as_uint(c1) & 1u) ? c2 : c1));
    }
    const float mean_c = fmaxf(mean, kFloor);
    const float sc = __fdiv_rn(1.0f, mean_c);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float f[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
      uint32_t part = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) part |= code_plus_one(f[i], sc) << (8 * (lane & 3) + 2 * i);
      part |= __shfl_xor_sync(0xFFFFFFFFu, part, 1);
      part |= __shfl_xor_sync(0xFFFFFFFFu, part, 2);
      if (ok[h] && (lane & 3) == 0) packed[(n * K + k0) / 16 + 8 * h + (lane >> 2)] = part;
    }
    if (lane == 0) D[blk] = mean_c;
  }
}

struct BlockFwdArgs {
  const int8_t* q;   // forward workspace: private-order int8 codes [M, K]
  const float* sx;   // [M]
  const uint32_t* packed;
  const float* D;    // [N, nb]
  float* y;          // [M, N]
  int64_t M, N, K;
  int64_t tiles_n;   // CTAs along the rows
  int nb, tm, rows_per_cta;
};

constexpr int kFwdWarps = 8;
constexpr int kStepWords = 256;  // words per warp step: 8 per lane, 16 blocks

__host__ __device__ inline size_t block_fwd_smem(int tm, int64_t K, int nb) {
  return (size_t)tm * (size_t)K + 4 * (size_t)tm * (size_t)nb + 4 * (size_t)tm;
}

template <int TM>
__global__ void __launch_bounds__(256) bl_block_scale_forward_kernel(BlockFwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile_m = (int64_t)blockIdx.x / a.tiles_n;
  const int64_t tile_n = (int64_t)blockIdx.x - tile_m * a.tiles_n;
  const int64_t t0 = tile_m * a.tm;
  const int tm = (int)std::min<int64_t>(a.tm, a.M - t0);
  const int K = (int)a.K, KW = K >> 4, nb = a.nb;
  int8_t* qs = reinterpret_cast<int8_t*>(smem);
  int32_t* bsum = reinterpret_cast<int32_t*>(smem + (size_t)a.tm * K);
  float* sxs = reinterpret_cast<float*>(smem + (size_t)a.tm * K + 4 * (size_t)a.tm * nb);

  // The tile's activation codes (tm rows of K bytes, contiguous) and scales.
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.q + t0 * a.K);
    uint4* dst = reinterpret_cast<uint4*>(qs);
    const int n16 = tm * KW;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = __ldg(src + i);
    if (threadIdx.x < tm) sxs[threadIdx.x] = __ldg(a.sx + t0 + threadIdx.x);
  }
  __syncthreads();
  // Per-token block sums of q (the codes are stored as code + 1).
  for (int p = warp; p < tm * nb; p += kFwdWarps) {
    const int m = p / nb, b = p - m * nb;
    const int k0 = b * kScaleBlock, cnt = min(kScaleBlock, K - k0);
    int s = 0;
    if (8 * lane < cnt) {
      const uint2 qq = *reinterpret_cast<const uint2*>(qs + (size_t)m * K + k0 + 8 * lane);
      s = __dp4a((int)qq.x, 0x01010101, s);
      s = __dp4a((int)qq.y, 0x01010101, s);
    }
    s = __reduce_add_sync(0xFFFFFFFFu, s);
    if (lane == 0) bsum[p] = s;
  }
  __syncthreads();

  // After the reduce-scatter below, lane L holds the sum of block
  // j = 2 * ((L >> 1) & 7) + (L >> 4) of the step; block j is read back from
  // lane 16 * (j & 1) + 2 * (j >> 1).
  const int jl = 2 * ((lane >> 1) & 7) + (lane >> 4);
  const bool b3 = (lane & 8) != 0, b2 = (lane & 4) != 0, b1 = (lane & 2) != 0;
  const int64_t row0 = tile_n * a.rows_per_cta;
  const int64_t row_end = std::min<int64_t>(row0 + a.rows_per_cta, a.N);
  for (int64_t r = row0 + warp; r < row_end; r += kFwdWarps) {
    const uint32_t* prow = a.packed + r * KW;
    const float* drow = a.D + r * nb;
    float yr[TM];
#pragma unroll
    for (int m = 0; m < TM; ++m) yr[m] = -0.0f;  // -0 + t == t for every t
    for (int w0 = 0; w0 < KW; w0 += kStepWords) {
      uint32_t wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int idx = w0 + lane + 32 * i;
        wv[i] = idx < KW ? __ldg(prow + idx) : 0u;
      }
      const int bb = (w0 >> 4) + jl;  // this lane's block after the reduction
      const float dv = bb < nb ? __ldg(drow + bb) : 0.0f;
      const int nblk = min(16, nb - (w0 >> 4));  // blocks present in this step
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        if (m < tm) {
          const int8_t* qrow = qs + (size_t)m * K;
          int av[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int idx = w0 + lane + 32 * i;
            int s = 0;
            if (idx < KW) {
              const uint4 qq = *reinterpret_cast<const uint4*>(qrow + 16 * idx);
              const uint32_t w = wv[i];
              s = __dp4a((int)(w & 0x03030303u), (int)qq.x, s);
              s = __dp4a((int)((w >> 2) & 0x03030303u), (int)qq.y, s);
              s = __dp4a((int)((w >> 4) & 0x03030303u), (int)qq.z, s);
              s = __dp4a((int)((w >> 6) & 0x03030303u), (int)qq.w, s);
            }
            av[i] = s;
          }
          // Reduce-scatter over the 16 lanes of each half-warp: 8 shuffles
          // leave lane L with the sum of av[(L >> 1) & 7] over its half.
          int c4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int send = b3 ? av[k] : av[k + 4];
            const int keep = b3 ? av[k + 4] : av[k];
            c4[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 8);
          }
          int c2[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int send = b2 ? c4[k] : c4[k + 2];
            const int keep = b2 ? c4[k + 2] : c4[k];
            c2[k] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 4);
          }
          int c1 = (b1 ? c2[1] : c2[0]) + __shfl_xor_sync(0xFFFFFFFFu, b1 ? c2[0] : c2[1], 2);
          c1 += __shfl_xor_sync(0xFFFFFFFFu, c1, 1);
          float t = 0.0f;
          if (bb < nb) t = rescale(c1 - bsum[m * nb + bb], sxs[m], dv);
          float yv = yr[m];
          for (int j = 0; j < nblk; ++j) yv = __fadd_rn(yv, __shfl_sync(0xFFFFFFFFu, t, 16 * (j & 1) + 2 * (j >> 1)));
          yr[m] = yv;
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < TM; ++m)
        if (m < tm) a.y[(t0 + m) * a.N + r] = yr[m];
    }
  }
}

template <int TM>
cudaError_t launch_block_forward_t(const BlockFwdArgs& a, unsigned grid, size_t smem, cudaStream_t stream) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(bl_block_scale_forward_kernel<TM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBlockFwdSmemMax);
    if (e != cudaSuccess) return e;
  }
  bl_block_scale_forward_kernel<TM><<<grid, kFwdWarps * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack_blocks(const float* W, int64_t N, int64_t K, uint32_t* packed, float* D, uint32_t* status,
                               cudaStream_t stream, int num_sms) {
  const int64_t total = N * scale_blocks(K);
  const int64_t want = (total + 7) / 8;
  const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)num_sms * 32);
  bl_block_scale_pack_kernel<<<grid, 256, 0, stream>>>(W, N, K, packed, D, status);
  return cudaGetLastError();
}

int block_forward_tile(int64_t M, int64_t K) {
  const int nb = (int)scale_blocks(K);
  int tm = (int)std::min<int64_t>(M, 16);
  while (tm > 1 && block_fwd_smem(tm, K, nb) > kBlockFwdSmemMax) --tm;
  return tm;
}

cudaError_t launch_forward_blocks(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                                  const void* ws, cudaStream_t stream, int num_sms) {
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  BlockFwdArgs a;
  a.q = reinterpret_cast<const int8_t*>(base + ws_q_off(M));
  a.sx = reinterpret_cast<const float*>(base + ws_sx_off(M));
  a.packed = packed;
  a.D = D;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.nb = (int)scale_blocks(K);
  a.tm = block_forward_tile(M, K);
  const int64_t tiles_m = (M + a.tm - 1) / a.tm;
  // Enough warps to keep every SM's loads in flight at one tile of tokens;
  // with several token tiles, more rows per CTA amortise the tile's load.
  int64_t rpw = (N + (int64_t)num_sms * 32 - 1) / ((int64_t)num_sms * 32);
  if (tiles_m > 1) rpw = std::max<int64_t>(rpw, 4);
  rpw = std::max<int64_t>(rpw, 1);
  a.rows_per_cta = (int)(rpw * kFwdWarps);
  a.tiles_n = (N + a.rows_per_cta - 1) / a.rows_per_cta;
  const int64_t grid = tiles_m * a.tiles_n;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  const size_t smem = block_fwd_smem(a.tm, K, a.nb);
  if (a.tm == 1) return launch_block_forward_t<1>(a, (unsigned)grid, smem, stream);
  if (a.tm <= 4) return launch_block_forward_t<4>(a, (unsigned)grid, smem, stream);
  return launch_block_forward_t<16>(a, (unsigned)grid, smem, stream);
}

}  // namespace bl
