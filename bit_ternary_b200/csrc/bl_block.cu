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
template <bool kBf16>
__device__ __noinline__ int compare_abs_sum(const void* __restrict__ wv, int cnt, double B) {
  uint32_t A[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) A[i] = 0u;
  for (int j = 0; j < cnt; ++j) {
    const float wj = kBf16 ? bf16_bits_to_float(__ldg(static_cast<const uint16_t*>(wv) + j))
                           : __ldg(static_cast<const float*>(wv) + j);
    const uint32_t b = __float_as_uint(wj) & 0x7FFFFFFFu;
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
template <bool kBf16>
__global__ void __launch_bounds__(256) bl_block_scale_pack_kernel(const void* __restrict__ W, int64_t N, int64_t K,
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
    const int64_t e0 = n * K + k0;  // first element of the block
    const void* src = kBf16 ? static_cast<const void*>(static_cast<const uint16_t*>(W) + e0)
                            : static_cast<const void*>(static_cast<const float*>(W) + e0);
    float4 v[2];
    bool ok[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = 128 * h + 4 * lane;
      ok[h] = c < cnt;
      v[h] = ok[h] ? load4<kBf16>(W, (e0 + c) >> 2) : make_float4(0.f, 0.f, 0.f, 0.f);
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
      if (lane == 0) cmp = compare_abs_sum<kBf16>(src, cnt, 0.5 * ((double)c1 + (double)c2) * (double)cnt);
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

// One warp step: the packed words of columns [16*w0, 16*w0 + 4096) of a row
// (8 per lane) and this lane's block scale after the reduction.
struct BlockStep {
  uint32_t w[8];
  float d;
};

__device__ __forceinline__ void load_step(BlockStep& st, const uint32_t* __restrict__ prow,
                                          const float* __restrict__ drow, int w0, int KW, int nb, int lane, int jl) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = w0 + lane + 32 * i;
    st.w[i] = idx < KW ? __ldg(prow + idx) : 0u;
  }
  const int bb = (w0 >> 4) + jl;
  st.d = bb < nb ? __ldg(drow + bb) : 0.0f;
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

  // This warp's rows are row0 + warp + 8*j; each is `steps` warp steps long.
  // The (row, step) units run in order with the next unit's loads in flight.
  // After the reduce-scatter below, lane L holds the sum of block
  // j = 2 * ((L >> 1) & 7) + (L >> 4) of a step; block j is read back from
  // lane 16 * (j & 1) + 2 * (j >> 1).
  const int jl = 2 * ((lane >> 1) & 7) + (lane >> 4);
  const int64_t row0 = tile_n * a.rows_per_cta;
  const int64_t row_end = std::min<int64_t>(row0 + a.rows_per_cta, a.N);
  const int64_t first = row0 + warp;
  const int nrows = first < row_end ? (int)((row_end - first + kFwdWarps - 1) / kFwdWarps) : 0;
  const int steps = (KW + kStepWords - 1) / kStepWords;
  BlockStep nxt;
  if (nrows > 0) load_step(nxt, a.packed + first * KW, a.D + first * nb, 0, KW, nb, lane, jl);

  // The weights above do not depend on the previous kernel in the stream (the
  // activation quantiser); its codes and scales are read only after it is done.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // The tile's activation codes (tm rows of K bytes, contiguous) and scales.
  // Plain loads: a read-only-path load (__ldg) counts as invariant memory and
  // may be hoisted above the wait, before the quantiser has written it.
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.q + t0 * a.K);
    uint4* dst = reinterpret_cast<uint4*>(qs);
    const int n16 = tm * KW;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = src[i];
    if (threadIdx.x < tm) sxs[threadIdx.x] = a.sx[t0 + threadIdx.x];
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

  const bool b3 = (lane & 8) != 0, b2 = (lane & 4) != 0, b1 = (lane & 2) != 0;
  float yr[TM];
#pragma unroll
  for (int m = 0; m < TM; ++m) yr[m] = -0.0f;  // -0 + t == t for every t
  int j = 0, st = 0;                              // current row index (of this warp) and step
  const int units = nrows * steps;
  for (int u = 0; u < units; ++u) {
    const BlockStep cur = nxt;
    const int64_t r = first + (int64_t)kFwdWarps * j;
    const int w0 = st * kStepWords;
    if (u + 1 < units) {
      const int jn = st + 1 == steps ? j + 1 : j, sn = st + 1 == steps ? 0 : st + 1;
      const int64_t rn = first + (int64_t)kFwdWarps * jn;
      load_step(nxt, a.packed + rn * KW, a.D + rn * nb, sn * kStepWords, KW, nb, lane, jl);
    }
    const int bb = (w0 >> 4) + jl;              // this lane's block after the reduction
    const int nblk = min(16, nb - (w0 >> 4));   // blocks present in this step
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
            const uint32_t w = cur.w[i];
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
        if (bb < nb) t = rescale(c1 - bsum[m * nb + bb], sxs[m], cur.d);
        float yv = yr[m];
        for (int jb = 0; jb < nblk; ++jb) yv = __fadd_rn(yv, __shfl_sync(0xFFFFFFFFu, t, 16 * (jb & 1) + 2 * (jb >> 1)));
        yr[m] = yv;
      }
    }
    if (++st == steps) {
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < TM; ++m)
          if (m < tm) a.y[(t0 + m) * a.N + r] = yr[m];
      }
#pragma unroll
      for (int m = 0; m < TM; ++m) yr[m] = -0.0f;
      st = 0;
      ++j;
    }
  }
}

// K % 256 == 0: every block is 16 whole words and block g of the flattened
// [N, nb] grid is the 64 bytes at word 16*g, so one lane owns one block (four
// 16-byte loads, no cross-lane reduction). A warp walks the blocks of its
// contiguous rows 32 at a time, with the next 32 blocks' loads in flight, and
// adds the terms of each row in order with shuffles. The activation codes sit
// in shared memory with block b's 16-byte chunk k at slot (k + b) mod 16, so
// that lanes on neighbouring blocks read different banks.
struct AlignedStep {
  uint4 w[4];
  float d;
};

__device__ __forceinline__ void load_aligned(AlignedStep& st, const uint32_t* __restrict__ packed,
                                             const float* __restrict__ D, int64_t g, bool ok) {
  const uint4* p = reinterpret_cast<const uint4*>(packed) + 4 * g;
#pragma unroll
  for (int i = 0; i < 4; ++i) st.w[i] = ok ? __ldg(p + i) : make_uint4(0u, 0u, 0u, 0u);
  st.d = ok ? __ldg(D + g) : 0.0f;
}

__device__ __forceinline__ int dot16(uint32_t w, const uint4& q, int acc) {
  acc = __dp4a((int)(w & 0x03030303u), (int)q.x, acc);
  acc = __dp4a((int)((w >> 2) & 0x03030303u), (int)q.y, acc);
  acc = __dp4a((int)((w >> 4) & 0x03030303u), (int)q.z, acc);
  return __dp4a((int)((w >> 6) & 0x03030303u), (int)q.w, acc);
}

template <int TM>
__global__ void __launch_bounds__(256) bl_block_scale_forward_aligned_kernel(BlockFwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t tile_m = (int64_t)blockIdx.x / a.tiles_n;
  const int64_t tile_n = (int64_t)blockIdx.x - tile_m * a.tiles_n;
  const int64_t t0 = tile_m * a.tm;
  const int tm = (int)std::min<int64_t>(a.tm, a.M - t0);
  const int K = (int)a.K, nb = a.nb;
  int8_t* qs = reinterpret_cast<int8_t*>(smem);
  int32_t* bsum = reinterpret_cast<int32_t*>(smem + (size_t)a.tm * K);
  float* sxs = reinterpret_cast<float*>(smem + (size_t)a.tm * K + 4 * (size_t)a.tm * nb);

  const int rpw = a.rows_per_cta / kFwdWarps;
  const int64_t wr0 = tile_n * a.rows_per_cta + (int64_t)warp * rpw;
  const int64_t wr1 = std::min<int64_t>(wr0 + rpw, a.N);
  const int64_t g0 = wr0 * nb, g1 = wr0 < wr1 ? wr1 * nb : g0;
  AlignedStep nxt;
  if (g0 < g1) load_aligned(nxt, a.packed, a.D, g0 + lane, g0 + lane < g1);

  // Weights and scales do not depend on the previous kernel in the stream
  // (the activation quantiser); its codes and scales are read after it is
  // done, with plain loads (a read-only-path load may be hoisted above this).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.q + t0 * a.K);
    uint4* dst = reinterpret_cast<uint4*>(qs);
    const int per_row = K >> 4;  // 16-byte chunks per token row
    const int n16 = tm * per_row;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) {
      const int m = i / per_row, c = i - m * per_row;
      const int b = c >> 4, k = c & 15;
      dst[m * per_row + 16 * b + ((k + b) & 15)] = src[i];
    }
    if (threadIdx.x < tm) sxs[threadIdx.x] = a.sx[t0 + threadIdx.x];
  }
  __syncthreads();
  for (int p = warp; p < tm * nb; p += kFwdWarps) {
    const int m = p / nb, b = p - m * nb;
    const uint2 qq = *reinterpret_cast<const uint2*>(qs + (size_t)m * K + 256 * b + 8 * lane);
    int s = __dp4a((int)qq.x, 0x01010101, 0);
    s = __dp4a((int)qq.y, 0x01010101, s);
    s = __reduce_add_sync(0xFFFFFFFFu, s);
    if (lane == 0) bsum[p] = s;
  }
  __syncthreads();

  float yr[TM];
#pragma unroll
  for (int m = 0; m < TM; ++m) yr[m] = -0.0f;  // -0 + t == t for every t
  int64_t n = wr0;                                // row of the next block to be added
  for (int64_t gb = g0; gb < g1; gb += 32) {
    const AlignedStep cur = nxt;
    if (gb + 32 < g1) load_aligned(nxt, a.packed, a.D, gb + 32 + lane, gb + 32 + lane < g1);
    const int nval = (int)std::min<int64_t>(32, g1 - gb);
    const int bl = (int)((gb % nb + lane) % nb);  // this lane's block within its row
    const unsigned ends = __ballot_sync(0xFFFFFFFFu, lane < nval && bl == nb - 1);
    const int sw = bl & 15;
#pragma unroll
    for (int m = 0; m < TM; ++m) {
      if (m < tm) {
        const uint4* qb = reinterpret_cast<const uint4*>(qs + (size_t)m * K + 256 * bl);
        int acc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t wi[4] = {cur.w[i].x, cur.w[i].y, cur.w[i].z, cur.w[i].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) acc = dot16(wi[j], qb[(4 * i + j + sw) & 15], acc);
        }
        const float t = lane < nval ? rescale(acc - bsum[m * nb + bl], sxs[m], cur.d) : 0.0f;
        float yv = yr[m];
        int64_t nn = n;
        for (int l = 0; l < nval; ++l) {
          yv = __fadd_rn(yv, __shfl_sync(0xFFFFFFFFu, t, l));
          if ((ends >> l) & 1u) {
            if (lane == 0) a.y[(t0 + m) * a.N + nn] = yv;
            yv = -0.0f;
            ++nn;
          }
        }
        yr[m] = yv;
      }
    }
    n += __popc(ends);
  }
}

template <int TM>
cudaError_t launch_block_forward_aligned_t(const BlockFwdArgs& a, unsigned grid, size_t smem, cudaStream_t stream) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(bl_block_scale_forward_aligned_kernel<TM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBlockFwdSmemMax);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFwdWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, bl_block_scale_forward_aligned_kernel<TM>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One token (M == 1), K % 256 == 0 and nb <= 32, in one launch: every CTA
// quantises the token itself (it is at most 32 KB of fp32). Lane l owns block l % nb of
// row l / nb of each warp step (floor(32 / nb) rows per step), so it keeps
// that block's 256 activation codes in registers for the whole launch and
// reads no shared memory. Each packed word is split into its four 2-bit
// classes by masks alone: byte j of (w & (3 << 2c) per byte) holds
// (code + 1) << 2c of column 4j + c, which the private activation order puts
// in byte j of the word c of the same 16-byte chunk. An unsigned x signed
// dp4a per class accumulates 4^c times the class sum; the four sums are
// recombined exactly by arithmetic shifts (each is an exact multiple).
struct BlockDecArgs {
  const void* x;    // [1, K] fp32 (or bf16 bit patterns), quantised by every CTA
  const uint32_t* packed;
  const float* D;   // [N, nb]
  float* y;         // [1, N]
  int64_t N;
  int K, nb, rows_per_warp;
};

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// NBT != 0 fixes the number of blocks per row at compile time (the per-row
// sum then unrolls); NBT == 0 reads it from the arguments.
template <int NBT, bool kBf16>
__global__ void __launch_bounds__(256, 2) bl_block_scale_decode_kernel(BlockDecArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb = NBT != 0 ? NBT : a.nb, R = 32 / nb;
  const int r = lane / nb, b = lane - r * nb;
  const bool active = r < R;
  const int64_t row0 = ((int64_t)blockIdx.x * kFwdWarps + warp) * a.rows_per_warp;
  const int64_t row1 = std::min<int64_t>(row0 + a.rows_per_warp, a.N);

  AlignedStep nxt;  // the first step's weights, requested before the quantiser runs
  {
    const int64_t row = row0 + r;
    const bool ok = active && row < row1;
    load_aligned(nxt, a.packed, a.D, ok ? row * nb + b : 0, ok);
  }
  // ActQuant of the token in every CTA (BitVLA section 1): max|x| over the
  // row, s_x = RN(127 / max(max|x|, 1e-5)), q = clamp(rint(RN(x * s_x))), the
  // codes stored in the private order (position 4c + j of each 16 holds
  // column 4j + c) in shared memory.
  __shared__ float red[kFwdWarps];
  __shared__ __align__(16) int8_t qs[kBlockDecMaxK];
  const int K4 = a.K >> 2;
  float amax = 0.0f;
  for (int i = threadIdx.x; i < K4; i += blockDim.x) {
    const float4 v = load4<kBf16>(a.x, i);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kFwdWarps; ++w) amax = fmaxf(amax, red[w]);
  const float sx = __fdiv_rn(kQmax, fmaxf(amax, kFloor));
  for (int g = threadIdx.x; g < (a.K >> 4); g += blockDim.x) {
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 f = load4<kBf16>(a.x, 4 * g + j);
      v[4 * j + 0] = quant_code(f.x, sx);
      v[4 * j + 1] = quant_code(f.y, sx);
      v[4 * j + 2] = quant_code(f.z, sx);
      v[4 * j + 3] = quant_code(f.w, sx);
    }
    uint32_t w4[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) word |= (uint32_t)(v[4 * j + c] & 0xFF) << (8 * j);
      w4[c] = word;
    }
    *reinterpret_cast<uint4*>(qs + 16 * g) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  __syncthreads();
  uint4 qv[16];
  const uint4* qb = reinterpret_cast<const uint4*>(qs + 256 * b);
#pragma unroll
  for (int k = 0; k < 16; ++k) qv[k] = qb[k];
  int bsum = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    bsum = __dp4a((int)qv[k].x, 0x01010101, bsum);
    bsum = __dp4a((int)qv[k].y, 0x01010101, bsum);
    bsum = __dp4a((int)qv[k].z, 0x01010101, bsum);
    bsum = __dp4a((int)qv[k].w, 0x01010101, bsum);
  }

  for (int64_t base = row0; base < row1; base += R) {
    const AlignedStep cur = nxt;
    if (base + R < row1) {
      const int64_t row = base + R + r;
      const bool ok = active && row < row1;
      load_aligned(nxt, a.packed, a.D, ok ? row * nb + b : 0, ok);
    }
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t wi[4] = {cur.w[i].x, cur.w[i].y, cur.w[i].z, cur.w[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t w = wi[j];
        const uint4& q = qv[4 * i + j];
        c0 = dp4a_us(w & 0x03030303u, q.x, c0);
        c1 = dp4a_us(w & 0x0C0C0C0Cu, q.y, c1);
        c2 = dp4a_us(w & 0x30303030u, q.z, c2);
        c3 = dp4a_us(w & 0xC0C0C0C0u, q.w, c3);
      }
    }
    const int acc = c0 + (c1 >> 2) + (c2 >> 4) + (c3 >> 6) - bsum;
    const int64_t row = base + r;
    const bool ok = active && row < row1;
    const float t = ok ? rescale(acc, sx, cur.d) : 0.0f;
    float yv = -0.0f;  // -0 + t == t for every t
    const int src = active ? r * nb : 0;
    if (NBT != 0) {
#pragma unroll
      for (int j = 0; j < (NBT != 0 ? NBT : 1); ++j) yv = __fadd_rn(yv, __shfl_sync(0xFFFFFFFFu, t, src + j));
    } else {
      for (int j = 0; j < nb; ++j) yv = __fadd_rn(yv, __shfl_sync(0xFFFFFFFFu, t, src + j));
    }
    if (ok && b == 0) a.y[row] = yv;
  }
}

template <int TM>
cudaError_t launch_block_forward_t(const BlockFwdArgs& a, unsigned grid, size_t smem, cudaStream_t stream) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(bl_block_scale_forward_kernel<TM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBlockFwdSmemMax);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFwdWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // Programmatic dependent launch: the weights start streaming while the
  // activation quantiser launched just before still runs.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, bl_block_scale_forward_kernel<TM>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Row sums of the activation codes per block, for the tensor-core route:
// bs[b * M + m] = sum of q[m, k] over block b's columns (the codes are stored
// as code + 1, so each block's contraction subtracts its own sum). One warp
// per (token, block); the private column order is a permutation inside
// groups of 16 columns, which never straddle blocks.
__global__ void __launch_bounds__(256) bl_block_scale_rowsum_kernel(const int8_t* __restrict__ q, int64_t M, int K,
                                                                    int nb, int32_t* __restrict__ bs) {
  const int lane = threadIdx.x & 31;
  const int64_t total = M * nb;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < total; p += warps) {
    const int64_t m = p / nb;
    const int b = (int)(p - m * nb);
    const int k0 = b * kScaleBlock, cnt = min(kScaleBlock, K - k0);
    int s = 0;
    if (8 * lane < cnt) {
      const uint2 qq = *reinterpret_cast<const uint2*>(q + m * K + k0 + 8 * lane);
      s = __dp4a((int)qq.x, 0x01010101, s);
      s = __dp4a((int)qq.y, 0x01010101, s);
    }
    s = __reduce_add_sync(0xFFFFFFFFu, s);
    if (lane == 0) bs[(int64_t)b * M + m] = s;
  }
}

}  // namespace

cudaError_t launch_pack_blocks(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D,
                               uint32_t* status, cudaStream_t stream, int num_sms) {
  const int64_t total = N * scale_blocks(K);
  const int64_t want = (total + 7) / 8;
  const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)num_sms * 32);
  if (bf16)
    bl_block_scale_pack_kernel<true><<<grid, 256, 0, stream>>>(W, N, K, packed, D, status);
  else
    bl_block_scale_pack_kernel<false><<<grid, 256, 0, stream>>>(W, N, K, packed, D, status);
  return cudaGetLastError();
}

int block_forward_tile(int64_t M, int64_t K) {
  const int nb = (int)scale_blocks(K);
  int tm = (int)std::min<int64_t>(M, 16);
  while (tm > 1 && block_fwd_smem(tm, K, nb) > kBlockFwdSmemMax) --tm;
  return tm;
}

cudaError_t launch_forward_blocks(const void* x, bool bf16, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                  const float* D, float* y, void* ws, cudaStream_t stream, int num_sms) {
  uint8_t* base = static_cast<uint8_t*>(ws);
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
  const bool aligned = (K % kScaleBlock) == 0;
  if (M == 1 && aligned && a.nb <= 32) {
    BlockDecArgs d;
    d.x = x;
    d.K = (int)K;
    d.packed = packed;
    d.D = D;
    d.y = y;
    d.N = N;
    d.nb = a.nb;
    const int R = 32 / a.nb;
    // About two CTAs of 8 warps per SM, each warp a whole number of steps.
    int64_t rpw = (N + (int64_t)num_sms * 16 - 1) / ((int64_t)num_sms * 16);
    rpw = (rpw + R - 1) / R * R;
    d.rows_per_warp = (int)rpw;
    const int64_t grid = (N + rpw * kFwdWarps - 1) / (rpw * kFwdWarps);
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kFwdWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    void (*kern)(BlockDecArgs) = nullptr;
#define BL_BDK(B)                                                                  \
  switch (a.nb) {                                                                  \
    case 4: kern = bl_block_scale_decode_kernel<4, B>; break;   /* K = 1024 */     \
    case 8: kern = bl_block_scale_decode_kernel<8, B>; break;   /* K = 2048 */     \
    case 10: kern = bl_block_scale_decode_kernel<10, B>; break; /* K = 2560 */     \
    case 12: kern = bl_block_scale_decode_kernel<12, B>; break; /* K = 3072 */     \
    case 27: kern = bl_block_scale_decode_kernel<27, B>; break; /* K = 6912 */     \
    default: kern = bl_block_scale_decode_kernel<0, B>; break;                     \
  }
    if (bf16) {
      BL_BDK(true)
    } else {
      BL_BDK(false)
    }
#undef BL_BDK
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, d);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  // Otherwise the activations are quantised once into the workspace (private
  // order), and the contraction launches as a programmatic dependent of that.
  cudaError_t eq = launch_act_quant(x, bf16, M, K, reinterpret_cast<int8_t*>(base + ws_q_off(M)),
                                    reinterpret_cast<float*>(base + ws_sx_off(M)),
                                    reinterpret_cast<int32_t*>(base + ws_rowsum_off(M)), true, stream,
                                    reinterpret_cast<uint32_t*>(base));
  if (eq != cudaSuccess) return eq;
  if (M >= kBlockGemmMinM) {
    // Tensor-core route: one GEMM per block over its K range (a 256-code
    // stage of the tcgen05 kernel is exactly one block), with the block's
    // column of D; the first block stores y, the others add their terms to it
    // in ascending order (the kernel's epilogue adds with one fp32 rounding).
    int32_t* bs = reinterpret_cast<int32_t*>(base + ws_forward_bytes(M, K));
    const int64_t nwarps = M * a.nb;
    const int64_t g = std::min<int64_t>((nwarps + 7) / 8, (int64_t)num_sms * 16);
    bl_block_scale_rowsum_kernel<<<(unsigned)g, 256, 0, stream>>>(a.q, M, (int)K, a.nb, bs);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    for (int b = 0; b < a.nb; ++b) {
      GemmSlice sl;
      sl.k0 = (int64_t)b * kScaleBlock;
      sl.kfull = K;
      sl.dstride = a.nb;
      sl.accumulate = b > 0;
      sl.rowsum = bs + (int64_t)b * M;
      const int64_t kc = std::min<int64_t>(kScaleBlock, K - sl.k0);
      e = launch_gemm_slice(M, N, kc, sl, packed, D + b, y, nullptr, ws, stream, num_sms);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const int64_t tiles_m = (M + a.tm - 1) / a.tm;
  // Enough warps to keep every SM's loads in flight at one tile of tokens;
  // with several token tiles, more rows per CTA amortise the tile's load. The
  // aligned kernel also wants at least 32 blocks (one per lane) per warp.
  int64_t rpw = (N + (int64_t)num_sms * 48 - 1) / ((int64_t)num_sms * 48);
  if (tiles_m > 1) rpw = std::max<int64_t>(rpw, 4);
  if (aligned) rpw = std::max<int64_t>(rpw, (32 + a.nb - 1) / a.nb);
  rpw = std::max<int64_t>(rpw, 1);
  a.rows_per_cta = (int)(rpw * kFwdWarps);
  a.tiles_n = (N + a.rows_per_cta - 1) / a.rows_per_cta;
  const int64_t grid = tiles_m * a.tiles_n;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  const size_t smem = block_fwd_smem(a.tm, K, a.nb);
  if (aligned) {
    if (a.tm == 1) return launch_block_forward_aligned_t<1>(a, (unsigned)grid, smem, stream);
    if (a.tm <= 4) return launch_block_forward_aligned_t<4>(a, (unsigned)grid, smem, stream);
    return launch_block_forward_aligned_t<16>(a, (unsigned)grid, smem, stream);
  }
  if (a.tm == 1) return launch_block_forward_t<1>(a, (unsigned)grid, smem, stream);
  if (a.tm <= 4) return launch_block_forward_t<4>(a, (unsigned)grid, smem, stream);
  return launch_block_forward_t<16>(a, (unsigned)grid, smem, stream);
}

}  // namespace bl
