// bl_decode.cu - decode BitLinear (M <= 16 tokens) for one or several
// independent BitLinears per launch: ActQuant (or RMSNorm + ActQuant) of the
// activations inside every CTA, the packed ternary weights streamed once from
// HBM through a shared-memory ring, an exact int32 contraction and the fp32
// rescale in the epilogue.
//
// The operation is the BitLinear product of "Core AI model zoo - BitVLA",
// section 2 (M=1 decode, arbitrary K with K % 16 == 0, any N, per-row scale
// D [N,1]), with the wrapper's ActQuant (section 1) done inside the kernel.
//
// Streaming. The packed weights are the only large stream (2 bits per weight).
// The unit of the stream is a tile: 16 consecutive rows, i.e. 16 * K/4
// contiguous bytes. Every CTA owns a contiguous, byte-balanced range of tiles
// over all problems of the launch (one CTA per SM). A producer warp keeps that
// range flowing through a byte ring in shared memory: one thread allocates a
// tile's bytes in the ring (first fit after the newest tile, wrapping to the
// start when the end is too short), issues one cp.async.bulk for it and hands
// it to the consumers through the tile's "full" mbarrier. A tile's bytes are
// given back when its "done" mbarrier fires, so up to the whole ring (about
// 90 KB, or 200 KB when one CTA holds the SM) is in flight at any time. The
// producer never reads activations, so it starts before griddepcontrol.wait:
// when launches are chained with programmatic dependent launch, a launch's
// weights stream while the previous launch still runs.
//
// Tasks. A tile is split into chunks of a few 256-code units; chunk j of tile i
// is one task, and consumer warp w takes every 8th task in (tile, chunk) order.
// A task's partial sums go to the tile's accumulator block in shared memory
// with shared atomics (exact integers, so the order does not matter); the warp
// that adds the tile's last chunk writes the outputs and releases the tile.
//
// Math. Lane (g, t) = (lane/4, lane%4) reads words 4t..4t+3 of each unit for
// rows g and g+8 of the tile. For class c in 0..3, word & (0x03030303 << 2c)
// leaves in byte b the value (code[4b+c]+1) << 2c: one AND gives four u8
// operands of mma.sync.m16n8k32 (u8 weights x s8 activations). One accumulator
// set per class, recombined exactly as acc0 + acc1/4 + acc2/16 + acc3/64, gives
// sum q*(code+1); subtracting sum q gives the signed result.
//
// Activations in shared memory. A token's codes are stored per 256-code unit;
// inside a unit, the 16 bytes of word w = 4t + 2h + j (codes 16w..16w+15, in
// the private order where position 4c+b holds column 4b+c) sit at byte
// 128h + 32t + 16j. Lane (g, t) then reads its 32 bytes of half h at 128h + 32t:
// the four lanes of a token cover 128 distinct bytes, and the row stride of
// 16 (mod 128) bytes moves the next token onto the other banks.
#include "bl_internal.h"

#include <atomic>
#include <cstring>

namespace bl {

constexpr int kDecConsumerWarps = 8;
constexpr int kDecConsumers = 32 * kDecConsumerWarps;
constexpr int kDecThreads = kDecConsumers + 32;  // + the producer warp
constexpr int kDecMaxGrid = 256;
constexpr int kDecRegGroups = 2;  // 16-column groups per thread held in registers by the quantiser
constexpr int kDecMaxUnitsPerTask = 5;
constexpr int kDecTok = kDecodeMaxGroup * 16;  // per-token state entries: problem * 16 + token

struct DecProblem {
  const void* x;        // fp32 / bf16 activations [M, K]; prepared mode: int8 codes, private order, [M, K]
  const float* sx_in;   // prepared mode: s_x [M]
  const int32_t* rs_in; // prepared mode: row sums [M]
  const uint32_t* packed;
  const float* D;
  float* y;
  int32_t* acc;
  int M;
  int N;
  int K;
  int wpr;       // packed words per row = K/16
  int nu;        // 256-code units per row = ceil(wpr / 16)
  int upt;       // units per task
  int nchunk;    // tasks per tile = ceil(nu / upt)
  int tiles;     // ceil(N / 16)
  int tile0;     // index of this problem's first tile in the launch
  int q_off;     // byte offset of this problem's codes in the shared activation block
  int q_stride;  // bytes per token row there (K rounded up to 256, + 16)
};

struct DecLaunch {
  DecProblem pr[kDecodeMaxGroup];
  const float* g;  // RMSNorm mode: norm weight [K] (one problem per launch)
  float eps;
  int nprob;
  int total_tiles;
  int ring_bytes;
  int q_bytes;
  uint32_t* err;
  int cta_start[kDecMaxGrid + 1];  // CTA c owns launch tiles [cta_start[c], cta_start[c+1])
};

// Shared memory past the ring and the activation codes.
__host__ __device__ constexpr int dec_fixed_bytes(int MT) {
  return kDecodeSlots * 16 * 8 * MT * 4   // s_acc
         + kDecodeSlots * 16 * 4          // s_D
         + 3 * kDecTok * 4              // s_sx, s_rs, s_amax
         + 2 * kDecodeSlots * 4           // s_cnt, s_off
         + 2 * kDecodeSlots * 8           // full, done
         + 16 * (8 + 4 + 4)             // RMSNorm: sums of squares, mean squares, flags
         + 16;                          // abort flag
}

__device__ __forceinline__ void dec_mma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void dec_bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
}

// Named barrier of the 8 consumer warps (the producer warp never joins it).
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumers) : "memory"); }

__device__ __forceinline__ int dec_problem_of(const DecLaunch& L, int gt) {
  int p = 0;
#pragma unroll 1
  while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
  return p;
}

// Byte offset, inside a unit, of the 16 codes of word w (see the file header).
__device__ __forceinline__ int dec_group_slot(int w) { return 128 * ((w >> 1) & 1) + 32 * (w >> 2) + 16 * (w & 1); }

// Shared-memory address of the 16 codes of group gi (columns 16gi..16gi+15) of token m.
__device__ __forceinline__ uint8_t* dec_q_group(uint8_t* sq, const DecProblem& P, int m, int gi) {
  return sq + P.q_off + m * P.q_stride + 256 * (gi >> 4) + dec_group_slot(gi & 15);
}

// Warp-aggregated shared atomics on per-token state; tok < 0 marks an idle
// lane. Called by all 32 lanes.
__device__ __forceinline__ void dec_amax(uint32_t* s_amax, int tok, float a) {
  const int t0 = __shfl_sync(0xFFFFFFFFu, tok, 0);
  if (__all_sync(0xFFFFFFFFu, tok == t0 || tok < 0)) {
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(a));  // a >= 0: bit order = value order
    if ((threadIdx.x & 31) == 0 && t0 >= 0) atomicMax(&s_amax[t0], m);
  } else if (tok >= 0) {
    atomicMax(&s_amax[tok], __float_as_uint(a));
  }
}

__device__ __forceinline__ void dec_rowsum(int32_t* s_rs, int tok, int s) {
  const int t0 = __shfl_sync(0xFFFFFFFFu, tok, 0);
  if (__all_sync(0xFFFFFFFFu, tok == t0 || tok < 0)) {
    const int sum = __reduce_add_sync(0xFFFFFFFFu, s);
    if ((threadIdx.x & 31) == 0 && t0 >= 0) atomicAdd(&s_rs[t0], sum);
  } else if (tok >= 0) {
    atomicAdd(&s_rs[tok], s);
  }
}

__device__ __forceinline__ float dec_absmax4(const float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// Quantise one 16-column group (float4 j holds columns 4j..4j+3) with scale
// sx, store its 16 codes in the private order, return their sum.
__device__ __forceinline__ int dec_quant_group(const float4 (&f)[4], float sx, uint8_t* dst) {
  int q[4][4];
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    q[j][0] = quant_code(f[j].x, sx);
    q[j][1] = quant_code(f[j].y, sx);
    q[j][2] = quant_code(f[j].z, sx);
    q[j][3] = quant_code(f[j].w, sx);
    sum += q[j][0] + q[j][1] + q[j][2] + q[j][3];
  }
  // Byte b of word r is column 4b + r: component r of float4 b.
  uint32_t w[4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
    w[r] = (uint32_t)(q[0][r] & 0xFF) | ((uint32_t)(q[1][r] & 0xFF) << 8) | ((uint32_t)(q[2][r] & 0xFF) << 16) |
           ((uint32_t)(q[3][r] & 0xFF) << 24);
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  return sum;
}

// Problems [pa, pb] of this CTA, flattened into 16-column groups: group gg
// belongs to problem p with pre[p - pa] <= gg < pre[p - pa + 1].
struct DecGroups {
  int pa, np, total;
  int pre[kDecodeMaxGroup + 1];
  __device__ __forceinline__ void locate(const DecLaunch& L, int gg, int& p, int& m, int& gi) const {
    int k = 0, base = 0;
#pragma unroll
    for (int i = 1; i < kDecodeMaxGroup; ++i)
      if (i < np && gg >= pre[i]) {
        k = i;
        base = pre[i];
      }
    p = pa + k;
    const int G = L.pr[p].K >> 4;
    const int local = gg - base;
    m = local / G;
    gi = local - m * G;
  }
};

template <int kX>
__device__ __forceinline__ void dec_load_group(const DecProblem& P, int m, int gi, float4 (&f)[4]) {
  const int64_t i4 = ((int64_t)m * P.K >> 2) + 4 * gi;
#pragma unroll
  for (int j = 0; j < 4; ++j) f[j] = load4<kX == kDecBf16>(P.x, i4 + j);
}

// ActQuant of every token of the CTA's problems into shared memory (fp32 or
// bf16 activations): per-token max|x| by shared atomics, then the codes, the
// scale s_x and the row sums. Run by the 256 consumer threads.
template <int kX>
__device__ void dec_quantise(const DecLaunch& L, const DecGroups& G, uint8_t* sq, float* s_sx, int32_t* s_rs,
                             uint32_t* s_amax) {
  const int tid = threadIdx.x;
  float4 f[kDecRegGroups][4];
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) {
    const int gg = tid + r * kDecConsumers;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      dec_load_group<kX>(L.pr[p], m, gi, f[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) {
    const int gg = tid + r * kDecConsumers;
    int tok = -1;
    float a = 0.0f;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      tok = p * 16 + m;
      a = fmaxf(fmaxf(dec_absmax4(f[r][0]), dec_absmax4(f[r][1])), fmaxf(dec_absmax4(f[r][2]), dec_absmax4(f[r][3])));
    }
    dec_amax(s_amax, tok, a);
  }
  // Groups beyond the registers: loaded now for the maximum, again for the codes.
  for (int base = kDecRegGroups * kDecConsumers; base < G.total; base += kDecConsumers) {
    const int gg = base + tid;
    int tok = -1;
    float a = 0.0f;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      float4 v[4];
      dec_load_group<kX>(L.pr[p], m, gi, v);
      tok = p * 16 + m;
      a = fmaxf(fmaxf(dec_absmax4(v[0]), dec_absmax4(v[1])), fmaxf(dec_absmax4(v[2]), dec_absmax4(v[3])));
    }
    dec_amax(s_amax, tok, a);
  }
  consumers_sync();  // every token's max|x| is complete
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) {
    const int gg = tid + r * kDecConsumers;
    int tok = -1, sum = 0;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      tok = p * 16 + m;
      const float sx = __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[tok]), kFloor));
      sum = dec_quant_group(f[r], sx, dec_q_group(sq, L.pr[p], m, gi));
      if (gi == 0) s_sx[tok] = sx;
    }
    dec_rowsum(s_rs, tok, sum);
  }
  for (int base = kDecRegGroups * kDecConsumers; base < G.total; base += kDecConsumers) {
    const int gg = base + tid;
    int tok = -1, sum = 0;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      float4 v[4];
      dec_load_group<kX>(L.pr[p], m, gi, v);
      tok = p * 16 + m;
      const float sx = __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[tok]), kFloor));
      sum = dec_quant_group(v, sx, dec_q_group(sq, L.pr[p], m, gi));
      if (gi == 0) s_sx[tok] = sx;
    }
    dec_rowsum(s_rs, tok, sum);
  }
}

// Prepared activations (int8 codes already in the private order, natural
// group order, row stride K; s_x and row sums): copied into the shared layout.
__device__ void dec_load_prepared(const DecLaunch& L, const DecGroups& G, uint8_t* sq, float* s_sx, int32_t* s_rs) {
  const int tid = threadIdx.x;
  for (int gg = tid; gg < G.total; gg += kDecConsumers) {
    int p, m, gi;
    G.locate(L, gg, p, m, gi);
    const DecProblem& P = L.pr[p];
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const int8_t*>(P.x) + (int64_t)m * P.K) + gi);
    *reinterpret_cast<uint4*>(dec_q_group(sq, P, m, gi)) = v;
  }
  for (int i = tid; i < G.np * 16; i += kDecConsumers) {
    const int p = G.pa + (i >> 4), m = i & 15;
    if (m < L.pr[p].M) {
      s_sx[p * 16 + m] = __ldg(L.pr[p].sx_in + m);
      s_rs[p * 16 + m] = __ldg(L.pr[p].rs_in + m);
    }
  }
}

// RMSNorm then ActQuant of every token of the launch's single problem ("BitNet-
// Embeddings I2_S guide", section 3.1): ms = mean(x^2) correctly rounded to
// fp32, r = RN(1/RN(sqrt(RN(ms + eps)))), n = RN(RN(x*r)*g), then the ActQuant
// of n. The squares are exact in fp64 and are summed in fp64 in whatever order
// the threads meet (shared atomics); any such sum of K non-negative terms is
// within (K-1)u/(1-(K-1)u) of the exact sum (u = 2^-53). Thread m widens
// RN64(sum/K) by (K+8)*2^-52 both ways with directed rounding; when the two
// ends round to different fp32 values (a rounding boundary inside the
// interval: a few tokens in a million) the token is summed again exactly in
// integer bins and divided with one correct rounding.
__device__ void dec_rms_quantise(const DecLaunch& L, const DecGroups& G, uint8_t* sq, float* s_sx, int32_t* s_rs,
                                 uint32_t* s_amax, double* s_ss, float* s_ms, int* s_flag,
                                 unsigned long long* bins) {
  const int tid = threadIdx.x;
  const DecProblem& P = L.pr[0];
  const int Gk = P.K >> 4;
  const float4* g4 = reinterpret_cast<const float4*>(L.g);
  float4 f[kDecRegGroups][4];
  // Sum of squares per token.
  for (int base = 0; base < G.total; base += kDecConsumers) {
    const int r = base / kDecConsumers;
    const int gg = base + tid;
    int tok = -1;
    double ss = 0.0;
    if (gg < G.total) {
      tok = gg / Gk;
      float4 v[4];
      dec_load_group<kDecF32>(P, tok, gg - tok * Gk, v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ss += (double)v[j].x * v[j].x + (double)v[j].y * v[j].y;
        ss += (double)v[j].z * v[j].z + (double)v[j].w * v[j].w;
        if (r < kDecRegGroups) {
#pragma unroll
          for (int rr = 0; rr < kDecRegGroups; ++rr)
            if (rr == r) f[rr][j] = v[j];
        }
      }
    }
    const int t0 = __shfl_sync(0xFFFFFFFFu, tok, 0);
    if (__all_sync(0xFFFFFFFFu, tok == t0 || tok < 0)) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      if ((tid & 31) == 0 && t0 >= 0) atomicAdd(&s_ss[t0], ss);
    } else if (tok >= 0) {
      atomicAdd(&s_ss[tok], ss);
    }
  }
  consumers_sync();
  if (tid < P.M) {
    const double qd = s_ss[tid] / (double)P.K;
    const double d = (double)(P.K + 8) * 2.220446049250313e-16;  // (K+8) * 2^-52
    const float flo = __double2float_rn(__dmul_rd(qd, 1.0 - d));
    const float fhi = __double2float_rn(__dmul_ru(qd, 1.0 + d));
    s_flag[tid] = flo != fhi;
    s_ms[tid] = flo;
  }
  consumers_sync();
  for (int m = 0; m < P.M; ++m) {
    if (!s_flag[m]) continue;  // uniform over the consumers
    for (int b = tid; b < kRmsBins; b += kDecConsumers) bins[b] = 0ull;
    consumers_sync();
    const float4* xr = reinterpret_cast<const float4*>(P.x) + ((int64_t)m * P.K >> 2);
    for (int i4 = tid; i4 < (P.K >> 2); i4 += kDecConsumers) {
      const float4 v = __ldg(xr + i4);
      rms_bins_add(bins, v.x);
      rms_bins_add(bins, v.y);
      rms_bins_add(bins, v.z);
      rms_bins_add(bins, v.w);
    }
    consumers_sync();
    if (tid == 0) s_ms[m] = mean_square_exact_f32(bins, (uint32_t)P.K);
    consumers_sync();
  }
  // n = RN(RN(x*r)*g); max|n| per token.
  auto normalise = [&](float4 (&v)[4], int tok, int gi) {
    const float rr = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(s_ms[tok], L.eps)));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 gw = __ldg(g4 + 4 * gi + j);
      v[j] = make_float4(__fmul_rn(__fmul_rn(v[j].x, rr), gw.x), __fmul_rn(__fmul_rn(v[j].y, rr), gw.y),
                         __fmul_rn(__fmul_rn(v[j].z, rr), gw.z), __fmul_rn(__fmul_rn(v[j].w, rr), gw.w));
    }
  };
  for (int base = 0; base < G.total; base += kDecConsumers) {
    const int r = base / kDecConsumers;
    const int gg = base + tid;
    int tok = -1;
    float a = 0.0f;
    if (gg < G.total) {
      tok = gg / Gk;
      const int gi = gg - tok * Gk;
      float4 v[4];
      if (r < kDecRegGroups) {
#pragma unroll
        for (int rr = 0; rr < kDecRegGroups; ++rr)
          if (rr == r) {
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = f[rr][j];
          }
      } else {
        dec_load_group<kDecF32>(P, tok, gi, v);
      }
      normalise(v, tok, gi);
      if (r < kDecRegGroups) {
#pragma unroll
        for (int rr = 0; rr < kDecRegGroups; ++rr)
          if (rr == r) {
#pragma unroll
            for (int j = 0; j < 4; ++j) f[rr][j] = v[j];
          }
      }
      a = fmaxf(fmaxf(dec_absmax4(v[0]), dec_absmax4(v[1])), fmaxf(dec_absmax4(v[2]), dec_absmax4(v[3])));
    }
    dec_amax(s_amax, tok, a);
  }
  consumers_sync();
  for (int base = 0; base < G.total; base += kDecConsumers) {
    const int r = base / kDecConsumers;
    const int gg = base + tid;
    int tok = -1, sum = 0;
    if (gg < G.total) {
      tok = gg / Gk;
      const int gi = gg - tok * Gk;
      float4 v[4];
      if (r < kDecRegGroups) {
#pragma unroll
        for (int rr = 0; rr < kDecRegGroups; ++rr)
          if (rr == r) {
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = f[rr][j];
          }
      } else {
        dec_load_group<kDecF32>(P, tok, gi, v);
        normalise(v, tok, gi);
      }
      const float sx = __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[tok]), kFloor));
      sum = dec_quant_group(v, sx, dec_q_group(sq, P, tok, gi));
      if (gi == 0) s_sx[tok] = sx;
    }
    dec_rowsum(s_rs, tok, sum);
  }
}

template <int MT, bool kAccOut, int kX>
__global__ void __launch_bounds__(kDecThreads, MT == 1 ? 2 : 1) bl_ternary_decode_kernel(const __grid_constant__ DecLaunch L) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint8_t* sq = smem + L.ring_bytes;
  int32_t* s_acc = reinterpret_cast<int32_t*>(sq + L.q_bytes);        // [slot][16 rows][8*MT tokens]
  float* s_D = reinterpret_cast<float*>(s_acc + kDecodeSlots * 16 * 8 * MT);  // [slot][16]
  float* s_sx = s_D + kDecodeSlots * 16;                                 // [problem * 16 + token]
  int32_t* s_rs = reinterpret_cast<int32_t*>(s_sx + kDecTok);
  uint32_t* s_amax = reinterpret_cast<uint32_t*>(s_rs + kDecTok);
  int32_t* s_cnt = reinterpret_cast<int32_t*>(s_amax + kDecTok);      // chunks added per slot
  uint32_t* s_off = reinterpret_cast<uint32_t*>(s_cnt + kDecodeSlots);  // ring offset per slot
  uint64_t* full = reinterpret_cast<uint64_t*>(s_off + kDecodeSlots);
  uint64_t* done = full + kDecodeSlots;
  double* s_ss = reinterpret_cast<double*>(done + kDecodeSlots);  // RMSNorm: [16] sums of squares
  float* s_ms = reinterpret_cast<float*>(s_ss + 16);              // [16] mean squares
  int* s_flag = reinterpret_cast<int*>(s_ms + 16);                // [16] exact path needed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(s_flag + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int t0 = L.cta_start[c];
  const int nt = L.cta_start[c + 1] - t0;

  // Dependents may be scheduled as soon as every CTA of this grid is running.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int s = 0; s < kDecodeSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < kDecodeSlots * 16 * 8 * MT; i += kDecThreads) s_acc[i] = 0;
  if (tid < kDecodeSlots) s_cnt[tid] = 0;
  if (tid < kDecTok) {
    s_amax[tid] = 0u;
    s_rs[tid] = 0;
  }
  if (tid < 16) s_ss[tid] = 0.0;
  __syncthreads();
  if (nt <= 0) return;

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint32_t R = (uint32_t)L.ring_bytes;
    uint32_t head = 0;  // end of the newest tile in the ring
    int tail = 0;       // oldest tile not yet seen released
    int issued = 0;
    bool ok = true;
    int p = dec_problem_of(L, t0);
    for (int i = 0; i < nt && ok; ++i) {
      const int gt = t0 + i;
      while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
      const DecProblem& P = L.pr[p];
      const int row0 = (gt - P.tile0) * 16;
      const int rows = P.N - row0 < 16 ? P.N - row0 : 16;
      const uint32_t bytes = (uint32_t)rows * (uint32_t)P.wpr * 4u;
      const uint32_t sz = (bytes + 127u) & ~127u;
      uint32_t off = 0;
      // First fit after the newest tile; otherwise wait for the oldest tile.
      for (;;) {
        if (tail == i) {
          off = 0;
          break;
        }
        if (i - tail < kDecodeSlots) {
          const uint32_t o = s_off[tail % kDecodeSlots];
          if (head > o) {  // live bytes [o, head)
            if (head + sz <= R) {
              off = head;
              break;
            }
            if (sz <= o) {
              off = 0;
              break;
            }
          } else if (head + sz <= o) {  // live bytes [o, R) and [0, head)
            off = head;
            break;
          }
        }
        if (!mbar_wait(&done[tail % kDecodeSlots], (uint32_t)(tail / kDecodeSlots) & 1u, abort_flag, L.err,
                       kDevTimeoutProducer)) {
          ok = false;
          break;
        }
        ++tail;
      }
      if (!ok) break;
      head = off + sz;
      const int s = i % kDecodeSlots;
      s_off[s] = off;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(P.packed + (int64_t)row0 * P.wpr);
      const uint32_t bulk = bytes & ~15u;
      if (bulk != bytes) {
        // 4..12 trailing bytes (a problem's last tile only): plain copies,
        // ordered for the readers by the barrier arrival below and for later
        // bulk writes to the same bytes by the proxy fence.
        for (uint32_t o = bulk; o < bytes; o += 4)
          *reinterpret_cast<uint32_t*>(ring + off + o) = __ldg(reinterpret_cast<const uint32_t*>(src + o));
        fence_proxy_async_smem();
      }
      mbar_arrive_expect_tx(&full[s], bulk);
      if (bulk) dec_bulk_g2s(ring + off, src, bulk, &full[s]);
      issued = i + 1;
    }
    if (!ok) {
      // Let the copies still in flight land before the CTA exits.
      for (int j = issued - kDecodeSlots > 0 ? issued - kDecodeSlots : 0; j < issued; ++j)
        mbar_wait(&full[j % kDecodeSlots], (uint32_t)(j / kDecodeSlots) & 1u, nullptr, L.err, kDevTimeoutDrain,
                  100000000ull);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  DecGroups G;
  G.pa = dec_problem_of(L, t0);
  G.np = dec_problem_of(L, t0 + nt - 1) - G.pa + 1;
  G.pre[0] = 0;
#pragma unroll
  for (int i = 0; i < kDecodeMaxGroup; ++i)
    G.pre[i + 1] = G.pre[i] + (i < G.np ? L.pr[G.pa + i].M * (L.pr[G.pa + i].K >> 4) : 0);
  G.total = G.pre[kDecodeMaxGroup];

  // The activations may be written by the grid this launch depends on: only
  // an L2 prefetch (no data is consumed) before the dependency wait.
  {
    const int esz = kX == kDecBf16 ? 2 : (kX == kDecPrepared ? 1 : 4);
    for (int i = 0; i < G.np; ++i) {
      const DecProblem& P = L.pr[G.pa + i];
      const int64_t bytes = (int64_t)P.M * P.K * esz;
      for (int64_t o = (int64_t)tid * 128; o < bytes; o += (int64_t)kDecConsumers * 128)
        prefetch_l2(static_cast<const uint8_t*>(P.x) + o);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && c == 0 && L.err != nullptr) *L.err = 0u;

  if (kX == kDecPrepared)
    dec_load_prepared(L, G, sq, s_sx, s_rs);
  else if (kX == kDecRms)
    dec_rms_quantise(L, G, sq, s_sx, s_rs, s_amax, s_ss, s_ms, s_flag,
                     reinterpret_cast<unsigned long long*>(sq + L.q_bytes - kRmsBins * 8));
  else
    dec_quantise<kX>(L, G, sq, s_sx, s_rs, s_amax);
  consumers_sync();  // codes, scales and row sums visible to every consumer warp

  const int g = lane >> 2, t = lane & 3;
  int p = G.pa;
  int task = 0;
  for (int i = 0; i < nt; ++i) {
    const int gt = t0 + i;
    while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
    const DecProblem& P = L.pr[p];
    const int C = P.nchunk;
    const int s = i % kDecodeSlots;
    const int row0 = (gt - P.tile0) * 16;
    const int rv = P.N - row0 < 16 ? P.N - row0 : 16;
    for (int j = (warp - task) & (kDecConsumerWarps - 1); j < C; j += kDecConsumerWarps) {
      if (!mbar_wait(&full[s], (uint32_t)(i / kDecodeSlots) & 1u, abort_flag, L.err, kDevTimeoutMma)) return;
      if (!kAccOut && j == 0 && lane < 16) s_D[s * 16 + lane] = lane < rv ? __ldg(P.D + row0 + lane) : 0.0f;
      const uint32_t* tile = reinterpret_cast<const uint32_t*>(ring + s_off[s]);
      const int wpr = P.wpr;
      // Rows past N are not in the ring: lanes on them read nothing.
      const bool aon = g < rv, bon = g + 8 < rv;
      const uint32_t* rowa = tile + (aon ? g : 0) * wpr + 4 * t;
      const uint32_t* rowb = tile + (bon ? g + 8 : 0) * wpr + 4 * t;
      const bool al = (wpr & 3) == 0;
      // Only lanes of existing tokens read activations (the other MMA
      // columns are never used).
      const uint8_t* qb[MT];
      bool qon[MT];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        qon[mt] = g + 8 * mt < P.M;
        qb[mt] = sq + P.q_off + (qon[mt] ? g + 8 * mt : 0) * P.q_stride + 32 * t;
      }
      int acc[4][MT][4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[cc][mt][k] = 0;
      const int ua = j * P.upt;
      const int ub = ua + P.upt < P.nu ? ua + P.upt : P.nu;
#pragma unroll 2
      for (int u = ua; u < ub; ++u) {
        uint32_t wa[4], wb[4];
        const int w0 = 16 * u + 4 * t;
        if (al && w0 + 4 <= wpr) {
          uint4 va = make_uint4(0u, 0u, 0u, 0u), vb = make_uint4(0u, 0u, 0u, 0u);
          if (aon) va = *reinterpret_cast<const uint4*>(rowa + 16 * u);
          if (bon) vb = *reinterpret_cast<const uint4*>(rowb + 16 * u);
          wa[0] = va.x;
          wa[1] = va.y;
          wa[2] = va.z;
          wa[3] = va.w;
          wb[0] = vb.x;
          wb[1] = vb.y;
          wb[2] = vb.z;
          wb[3] = vb.w;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const bool in = w0 + k < wpr;  // words past the row belong to the next row: zero
            wa[k] = in && aon ? rowa[16 * u + k] : 0u;
            wb[k] = in && bon ? rowb[16 * u + k] : 0u;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 Q[MT][2];
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            Q[mt][0] = make_uint4(0u, 0u, 0u, 0u);
            Q[mt][1] = make_uint4(0u, 0u, 0u, 0u);
            if (qon[mt]) {
              const uint8_t* qp = qb[mt] + 256 * u + 128 * h;
              Q[mt][0] = *reinterpret_cast<const uint4*>(qp);
              Q[mt][1] = *reinterpret_cast<const uint4*>(qp + 16);
            }
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t mask = 0x03030303u << (2 * cc);
            const uint32_t a0 = wa[2 * h] & mask, a2 = wa[2 * h + 1] & mask;
            const uint32_t a1 = wb[2 * h] & mask, a3 = wb[2 * h + 1] & mask;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const uint32_t b0 = cc == 0 ? Q[mt][0].x : (cc == 1 ? Q[mt][0].y : (cc == 2 ? Q[mt][0].z : Q[mt][0].w));
              const uint32_t b1 = cc == 0 ? Q[mt][1].x : (cc == 1 ? Q[mt][1].y : (cc == 2 ? Q[mt][1].z : Q[mt][1].w));
              dec_mma(acc[cc][mt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }
      // Partial sums of this chunk into the tile's block: class c holds
      // 4^c * sum q*(code+1), an exact multiple of 4^c.
      int32_t* blk = s_acc + s * 16 * 8 * MT;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int tok = 8 * mt + 2 * t + (k & 1);
          if (tok < P.M) {
            const int v = acc[0][mt][k] + (acc[1][mt][k] >> 2) + (acc[2][mt][k] >> 4) + (acc[3][mt][k] >> 6);
            atomicAdd(blk + (g + 8 * (k >> 1)) * 8 * MT + tok, v);
          }
        }
      __syncwarp();
      __threadfence_block();
      int last = 0;
      if (lane == 0) last = atomicAdd(&s_cnt[s], 1) == C - 1;
      last = __shfl_sync(0xFFFFFFFFu, last, 0);
      if (last) {
        // Every chunk of the tile is in: outputs, then release the tile.
        __threadfence_block();
        for (int idx = lane; idx < 16 * P.M; idx += 32) {
          const int tok = idx >> 4, r = idx & 15;
          if (r < rv) {
            const int a = blk[r * 8 * MT + tok] - s_rs[p * 16 + tok];
            const int64_t o = (int64_t)tok * P.N + row0 + r;
            if (kAccOut)
              P.acc[o] = a;
            else
              P.y[o] = rescale(a, s_sx[p * 16 + tok], s_D[s * 16 + r]);
          }
        }
        __syncwarp();
        for (int k = lane; k < 16 * 8 * MT; k += 32) blk[k] = 0;
        if (lane == 0) s_cnt[s] = 0;
        __syncwarp();
        __threadfence_block();
        if (lane == 0) mbar_arrive(&done[s]);
      }
    }
    task += C;
  }
}

template <int MT, bool kAccOut, int kX>
static cudaError_t launch_decode_t(const DecLaunch& L, int grid, size_t smem, bool pdl, cudaStream_t stream) {
  auto kern = bl_ternary_decode_kernel<MT, kAccOut, kX>;
  // The shared-memory limit is raised once per device for each instantiation.
  static std::atomic<int> raised[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || raised[dev].load(std::memory_order_relaxed) < (int)smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecodeSmemMax);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev].store((int)kDecodeSmemMax, std::memory_order_relaxed);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, L);
}

int64_t decode_q_stride(int64_t K) { return ((K + 255) / 256) * 256 + 16; }

static int64_t round128(int64_t v) { return (v + 127) / 128 * 128; }

static int64_t tile_bytes_max(int64_t K) { return round128(16 * (K / 4)); }

// Shared-memory plan of a launch: ring bytes and total, or false when the
// calls do not fit (then they take the tensor-core path).
// q_total includes the RMSNorm mode's exact-sum bins, which follow the codes.
static bool decode_plan(int64_t q_total, int64_t tile_max, int MT, int64_t* ring, int64_t* total) {
  const int64_t fixed = dec_fixed_bytes(MT);
  // Two CTAs per SM when three tiles fit beside the codes (a launch's CTAs
  // then leave room on every SM for the next launch's), else one.
  const int64_t budgets[2] = {kDecodeSmemShared, kDecodeSmemMax};
  const int64_t want_tiles[2] = {3, 2};
  for (int b = 0; b < 2; ++b) {
    const int64_t r = (budgets[b] - q_total - fixed) / 128 * 128;
    if (r >= want_tiles[b] * tile_max) {
      *ring = r;
      *total = r + q_total + fixed;
      return true;
    }
  }
  return false;
}

bool decode_group_fits(const DecCall* calls, int n) {
  if (n < 1 || n > kDecodeMaxGroup) return false;
  int64_t q = 0, tmax = 0, maxM = 0;
  for (int i = 0; i < n; ++i) {
    if (calls[i].M < 1 || calls[i].M > kDecodeMaxM) return false;
    q += round128(calls[i].M * decode_q_stride(calls[i].K));
    const int64_t tb = tile_bytes_max(calls[i].K);
    tmax = tb > tmax ? tb : tmax;
    maxM = calls[i].M > maxM ? calls[i].M : maxM;
  }
  int64_t ring = 0, total = 0;
  return decode_plan(q, tmax, maxM <= 8 ? 1 : 2, &ring, &total);
}

bool decode_fits(int64_t M, int64_t K, bool rms) {
  if (M < 1 || M > kDecodeMaxM) return false;
  int64_t ring = 0, total = 0;
  const int64_t q = round128(M * decode_q_stride(K)) + (rms ? kRmsBins * 8 : 0);
  return decode_plan(q, tile_bytes_max(K), M <= 8 ? 1 : 2, &ring, &total);
}

// Bytes of launch tile gt (rows x K/4, rounded up to 128).
static int64_t host_tile_bytes(const DecLaunch& L, int gt) {
  int p = 0;
  while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
  const DecProblem& P = L.pr[p];
  const int64_t row0 = (int64_t)(gt - P.tile0) * 16;
  const int64_t rows = P.N - row0 < 16 ? P.N - row0 : 16;
  return round128(rows * P.wpr * 4);
}

// Split the launch's tiles into `grid` contiguous ranges of about equal bytes,
// at least one tile each.
static void partition_by_bytes(DecLaunch& L, int grid) {
  int64_t total = 0;
  for (int gt = 0; gt < L.total_tiles; ++gt) total += host_tile_bytes(L, gt);
  int64_t acc = 0;
  int cta = 0, start = 0;
  L.cta_start[0] = 0;
  for (int gt = 0; gt < L.total_tiles; ++gt) {
    const int64_t tb = host_tile_bytes(L, gt);
    const int64_t target = total * (cta + 1) / grid;
    if (cta + 1 < grid && gt > start && acc + tb / 2 > target && L.total_tiles - gt >= grid - cta - 1) {
      L.cta_start[++cta] = gt;
      start = gt;
    }
    acc += tb;
  }
  for (int k = cta + 1; k <= grid; ++k) L.cta_start[k] = L.total_tiles;
}

cudaError_t launch_decode(const DecCall* calls, int n, int input, const float* g, float eps, uint32_t* err, bool pdl,
                          cudaStream_t stream, int num_sms) {
  if (n < 1 || n > kDecodeMaxGroup) return cudaErrorInvalidValue;
  if ((input == kDecRms || input == kDecPrepared) && n != 1) return cudaErrorInvalidValue;
  DecLaunch L;
  std::memset(&L, 0, sizeof(L));
  int64_t maxM = 0, q = 0, tmax = 0;
  int tiles = 0;
  for (int i = 0; i < n; ++i) {
    DecProblem& P = L.pr[i];
    P.x = calls[i].x;
    P.sx_in = calls[i].sx;
    P.rs_in = calls[i].rs;
    P.packed = calls[i].packed;
    P.D = calls[i].D;
    P.y = calls[i].y;
    P.acc = calls[i].acc;
    P.M = (int)calls[i].M;
    P.N = (int)calls[i].N;
    P.K = (int)calls[i].K;
    P.wpr = P.K / 16;
    P.nu = (P.wpr + 15) / 16;
    P.tiles = (P.N + 15) / 16;
    P.tile0 = tiles;
    P.q_stride = (int)decode_q_stride(P.K);
    P.q_off = (int)q;
    q += round128((int64_t)P.M * P.q_stride);
    tiles += P.tiles;
    maxM = calls[i].M > maxM ? calls[i].M : maxM;
    const int64_t tb = tile_bytes_max(calls[i].K);
    tmax = tb > tmax ? tb : tmax;
    if (calls[i].M < 1 || calls[i].M > kDecodeMaxM || calls[i].N < 1) return cudaErrorInvalidValue;
  }
  const int MT = maxM <= 8 ? 1 : 2;
  if (input == kDecRms) q += kRmsBins * 8;  // exact-sum bins after the codes
  int64_t ring = 0, total = 0;
  if (!decode_plan(q, tmax, MT, &ring, &total)) return cudaErrorInvalidValue;
  L.nprob = n;
  L.total_tiles = tiles;
  L.ring_bytes = (int)ring;
  L.q_bytes = (int)q;
  L.err = err;
  L.g = g;
  L.eps = eps;
  int grid = tiles < num_sms ? tiles : num_sms;
  if (grid > kDecMaxGrid) grid = kDecMaxGrid;
  partition_by_bytes(L, grid);
  // Units per task: about eight tasks per warp-sized share of a CTA's tiles
  // for short launches (latency), up to kDecMaxUnitsPerTask for long ones.
  const double tiles_per_cta = (double)tiles / grid;
  for (int i = 0; i < n; ++i) {
    DecProblem& P = L.pr[i];
    int upt = (int)((P.nu * tiles_per_cta + kDecConsumerWarps - 1) / kDecConsumerWarps);
    upt = upt < 1 ? 1 : (upt > kDecMaxUnitsPerTask ? kDecMaxUnitsPerTask : upt);
    if (upt > P.nu) upt = P.nu;
    P.upt = upt;
    P.nchunk = (P.nu + upt - 1) / upt;
  }
  const bool accout = calls[0].acc != nullptr;
  for (int i = 1; i < n; ++i)
    if ((calls[i].acc != nullptr) != accout) return cudaErrorInvalidValue;  // one output kind per launch
#define BL_DEC(MTV, AO, XM) \
  if (MT == MTV && accout == AO && input == XM) return launch_decode_t<MTV, AO, XM>(L, grid, (size_t)total, pdl, stream);
  BL_DEC(1, false, kDecF32)
  BL_DEC(1, true, kDecF32)
  BL_DEC(2, false, kDecF32)
  BL_DEC(2, true, kDecF32)
  BL_DEC(1, false, kDecBf16)
  BL_DEC(1, true, kDecBf16)
  BL_DEC(2, false, kDecBf16)
  BL_DEC(2, true, kDecBf16)
  BL_DEC(1, false, kDecPrepared)
  BL_DEC(2, false, kDecPrepared)
  BL_DEC(1, false, kDecRms)
  BL_DEC(2, false, kDecRms)
#undef BL_DEC
  return cudaErrorInvalidValue;
}

}  // namespace bl
