// bl_gemv.cu - decode GEMV (M <= 16 tokens) with ActQuant fused in, for one
// or several independent BitLinears per launch.
//
// The operation is the BitLinear product of "Core AI model zoo - BitVLA",
// section 2 (M=1 decode, arbitrary K with K % 16 == 0, any N, per-row scale
// D [N,1]), with the wrapper's ActQuant (section 1) done inside the kernel.
//
// Design (B200). The packed weights are the only large stream (2 bits per
// weight). The grid is persistent: CTA c owns a contiguous, byte-balanced
// range of 16-row tiles over all problems of the launch. One thread issues
// cp.async.bulk copies of whole tiles (16 rows x K/4 bytes, contiguous in
// memory) into shared memory the moment the CTA starts, and the row scales D
// follow by cp.async, so every byte of weights the CTA needs is in flight
// before x is read. A CTA needs at most ~100 KB of shared memory and 64
// registers per thread for M <= 8, so two CTAs fit on an SM: under
// programmatic dependent launch the next launch's CTAs become resident while
// this one runs and stream their weights in the meantime; activations are read
// only after griddepcontrol.wait.
//
// Quantise. Every CTA quantises x itself (x is small and L2-resident): a
// thread takes one 16-column group, the per-token absmax is a warp reduction
// plus one shared atomic per warp, and the codes are written as one 16-byte
// store in the kernel-private column order (inside every 16 columns, position
// 4c+b holds column 4b+c). Wider activations stride over float4s instead.
//
// Math. Lane (g, t) = (lane/4, lane%4) of a warp takes words 4t..4t+3 of each
// 256-code unit for rows g and g+8 of a tile; warp w takes a contiguous range
// of (tile, unit) tasks, so it flushes its sums to the tile's shared block once
// per tile. Unpacking is one AND per 4 codes: for class c in 0..3,
// word & (0x03030303 << 2c) leaves, in byte b, (code[4b+c]+1) << 2c. Those
// bytes feed mma.sync.m16n8k32 (u8 weights x s8 activations) with one
// accumulator set per class, recombined exactly as acc0 + acc1/4 + acc2/16 +
// acc3/64; only lanes of existing tokens load activations (the other MMA
// columns are never read). sum q*(code+1) - sum q gives the signed result.
#include "bl_internal.h"

#include <cstring>

namespace bl {

constexpr int kGemvWarps = 16;  // warps per CTA: enough independent work to hide latency
constexpr int kGemvThreads = 32 * kGemvWarps;
constexpr int kGemvMaxGrid = 256;

struct GemvProblem {
  const void* x;  // fp32, or bf16 bit patterns (kBf16)
  const uint32_t* packed;
  const float* D;
  float* y;
  int32_t* acc;
  int M;
  int N;
  int K;
  int wpr;       // packed words per row = K/16
  int n_units;   // ceil(wpr / 16)
  int tiles;     // ceil(N / 16)
  int tile0;     // index of this problem's first tile in the launch
  int q_stride;  // shared bytes per token row of quantised activations
};

struct GemvLaunch {
  GemvProblem pr[kGemvMaxGroup];
  int nprob;
  int total_tiles;
  int stage_bytes;  // bytes of one tile slot of the double-buffered mode (widest problem)
  int round_tiles;  // tile slots per round buffer
  int nbuf;         // 1: all of a CTA's tiles in flight, packed by size; 2: double-buffered rounds
  int buf_bytes;    // capacity of one round buffer
  int q_bytes;
  int xs_bytes;     // staging of fp32 activations between the absmax and the quantise
  uint32_t* err;
  int cta_start[kGemvMaxGrid + 1];  // CTA c owns launch tiles [cta_start[c], cta_start[c+1])
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ int problem_of(const GemvLaunch& L, int gt) {
  int p = 0;
#pragma unroll 1
  while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
  return p;
}

// Bytes of launch tile `gt` in shared memory (rows x K/4, rounded up to 128).
__device__ __forceinline__ uint32_t tile_slot_bytes(const GemvLaunch& L, int gt) {
  const GemvProblem& P = L.pr[problem_of(L, gt)];
  const int row0 = (gt - P.tile0) * 16;
  const int rows = P.N - row0 < 16 ? P.N - row0 : 16;
  return ((uint32_t)rows * (uint32_t)P.wpr * 4u + 127u) & ~127u;
}

// Start the copy of launch tile `gt` into shared memory (one thread). A tile
// is rows_valid x K/4 contiguous bytes. Whole 16-byte chunks go by bulk copy;
// a remainder of 4..12 bytes (only possible on a problem's last tile) is
// copied with plain loads before the barrier's arrival, which orders it for
// the readers.
__device__ __forceinline__ void issue_tile(const GemvLaunch& L, int gt, uint8_t* dst, uint64_t* bar) {
  const GemvProblem& P = L.pr[problem_of(L, gt)];
  const int lt = gt - P.tile0;
  const int row0 = lt * 16;
  const int rows = P.N - row0 < 16 ? P.N - row0 : 16;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(P.packed + (int64_t)row0 * P.wpr);
  const uint32_t bytes = (uint32_t)rows * (uint32_t)P.wpr * 4u;
  const uint32_t bulk = bytes & ~15u;
  for (uint32_t o = bulk; o < bytes; o += 4)
    *reinterpret_cast<uint32_t*>(dst + o) = __ldg(reinterpret_cast<const uint32_t*>(src + o));
  mbar_arrive_expect_tx(bar, bulk);
  if (bulk) bulk_g2s(dst, src, bulk, bar);
}

// Activations of one problem are quantised per CTA into shared memory, in the
// kernel-private column order, with per-token scale s_x and sum of codes.
// Threads stride over the float4s of the row-major [M, K] block twice
// (absmax, then quantise; the second pass hits L1), kXBatch float4 loads in
// flight per thread. Element 4j+e of a
// 16-column group (float4 j, lane e) goes to byte 4e+j of the group: the
// order perm16 describes.

constexpr int kXBatch = 4;

__device__ __forceinline__ float absmax4(const float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// Warp-aggregated shared atomics. The lanes of a warp usually hold one token,
// and then one lane updates for all of them. tok < 0 marks an idle lane; idle
// lanes are always the last ones of the warp. Called by all 32 lanes.
__device__ __forceinline__ void warp_amax(uint32_t* s_amax, int tok, float a) {
  const int t0 = __shfl_sync(0xFFFFFFFFu, tok, 0);
  if (__all_sync(0xFFFFFFFFu, tok == t0 || tok < 0)) {
    // non-negative floats order as their bit patterns
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(a));
    if ((threadIdx.x & 31) == 0 && t0 >= 0) atomicMax(&s_amax[t0], m);
  } else if (tok >= 0) {
    atomicMax(&s_amax[tok], __float_as_uint(a));
  }
}

__device__ __forceinline__ void warp_rowsum(int32_t* s_rs, int tok, int s) {
  const int t0 = __shfl_sync(0xFFFFFFFFu, tok, 0);
  if (__all_sync(0xFFFFFFFFu, tok == t0 || tok < 0)) {
    const int sum = __reduce_add_sync(0xFFFFFFFFu, s);
    if ((threadIdx.x & 31) == 0 && t0 >= 0) atomicAdd(&s_rs[t0], sum);
  } else if (tok >= 0) {
    atomicAdd(&s_rs[tok], s);
  }
}

// int8 code clamp(rint(RN(x*s_x)), -128, 127), rounding by the addition of
// 1.5*2^23: for |v| < 2^22 the fp32 sum v + 1.5*2^23 lies in [2^23, 2^24),
// where the spacing is 1, so the addition itself rounds v to the nearest
// integer, ties to even, exactly as rint does; the integer is the difference
// of the bit patterns. Larger or non-finite products take the conversion
// instruction, so every input gives the same code as quant_i8.
__device__ __forceinline__ int quant_i8_fast(float x, float s_x) {
  const float v = __fmul_rn(x, s_x);
  int q;
  if (fabsf(v) < 4194304.0f)
    q = __float_as_int(__fadd_rn(v, 12582912.0f)) - 0x4B400000;
  else
    q = __float2int_rn(v);
  return q < -128 ? -128 : (q > 127 ? 127 : q);
}

// Quantise one float4 (token m, float4 column c4) into shared memory; returns
// the sum of its four codes.
__device__ __forceinline__ int quant_store4(uint8_t* sq, int q_stride, int m, int c4, const float4 f, float sx) {
  const int q0 = quant_i8_fast(f.x, sx), q1 = quant_i8_fast(f.y, sx), q2 = quant_i8_fast(f.z, sx),
            q3 = quant_i8_fast(f.w, sx);
  uint8_t* dst = sq + (int64_t)m * q_stride + 16 * (c4 >> 2) + (c4 & 3);
  dst[0] = (uint8_t)q0;
  dst[4] = (uint8_t)q1;
  dst[8] = (uint8_t)q2;
  dst[12] = (uint8_t)q3;
  return q0 + q1 + q2 + q3;
}

__device__ __forceinline__ float token_scale(const uint32_t* s_amax, int m) {
  return __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[m]), kFloor));
}

// 4-byte asynchronous copy global -> shared (row scales), waited for with
// cp.async.wait_all before the outputs are written.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
               "l"(__cvta_generic_to_global(src))
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Add a warp's partial sums for one 16-row tile into the tile's shared block.
// The four classes are recombined exactly: class c holds 4^c * sum q*(code+1).
template <int MT, int DA>
__device__ __forceinline__ void flush_tile(const int (&acc)[4][DA][MT][4], int* dst, int g, int t) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
      for (int d = 0; d < DA; ++d) {
        c0 += acc[0][d][mt][q];
        c1 += acc[1][d][mt][q];
        c2 += acc[2][d][mt][q];
        c3 += acc[3][d][mt][q];
      }
      const int v = c0 + (c1 >> 2) + (c2 >> 4) + (c3 >> 6);
      const int row = g + 8 * (q >> 1), tok = 8 * mt + 2 * t + (q & 1);
      atomicAdd(dst + row * 8 * MT + tok, v);
    }
}

template <int MT, bool kAccOut, bool kBf16>
__global__ void __launch_bounds__(kGemvThreads, MT == 1 ? 2 : 1) gemv_kernel(const __grid_constant__ GemvLaunch L) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int RT = L.round_tiles;                                           // tiles per round buffer
  uint8_t* bufs = smem;                                                   // [nbuf][buf_bytes]
  uint8_t* sq = smem + (size_t)L.nbuf * L.buf_bytes;
  float4* s_xs = reinterpret_cast<float4*>(sq + L.q_bytes);              // [xs_bytes / 16]
  // Per-token state in two sets: consecutive problems of a CTA alternate.
  float* s_sx = reinterpret_cast<float*>(sq + L.q_bytes + L.xs_bytes);    // [2][16]
  int32_t* s_rs = reinterpret_cast<int32_t*>(s_sx + 32);                  // [2][16]
  uint32_t* s_amax = reinterpret_cast<uint32_t*>(s_rs + 32);              // [2][16]
  float* s_D = reinterpret_cast<float*>(s_amax + 32);                     // [RT * 16] row scales of the round
  int32_t* s_acc = reinterpret_cast<int32_t*>(s_D + (size_t)RT * 16);     // [RT][16 rows][8*MT tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_acc + (size_t)RT * 16 * 8 * MT);  // [nbuf][RT]
  uint32_t* s_off = reinterpret_cast<uint32_t*>(full + (size_t)L.nbuf * RT);       // [nbuf][RT] tile offsets
  volatile int* abort_flag = reinterpret_cast<volatile int*>(s_off + (size_t)L.nbuf * RT);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int c = blockIdx.x;
  const int t0 = L.cta_start[c];
  const int nt = L.cta_start[c + 1] - t0;
  const int nrounds = (nt + RT - 1) / RT;

  if (tid == 0) {
    for (int s = 0; s < L.nbuf * RT; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid < 32) {
    s_amax[tid] = 0u;
    s_rs[tid] = 0;
  }
  __syncthreads();
  // Issue every copy of round r into buffer r % nbuf (one thread). Tiles are
  // packed by size; the offset table is written before each tile's barrier
  // arrival, so a reader that has waited on the barrier sees it.
  auto issue_round = [&](int r) {
    const int b = r % L.nbuf;
    const int a = r * RT, e = (a + RT < nt) ? a + RT : nt;
    uint32_t off = 0;
    for (int i = a; i < e; ++i) {
      s_off[b * RT + (i - a)] = off;
      issue_tile(L, t0 + i, bufs + (size_t)b * L.buf_bytes + off, &full[b * RT + (i - a)]);
      off += tile_slot_bytes(L, t0 + i);
    }
  };
  // Row scales D of round r's tiles into s_D (all threads). The int32
  // accumulator output has no D.
  auto load_D = [&](int r) {
    if (kAccOut) return;
    const int a = r * RT, e = (a + RT < nt) ? a + RT : nt;
    for (int i = tid; i < (e - a) * 16; i += kGemvThreads) {
      const int gt = t0 + a + (i >> 4);
      const GemvProblem& P = L.pr[problem_of(L, gt)];
      const int row = (gt - P.tile0) * 16 + (i & 15);
      if (row < P.N && P.D != nullptr) cp_async4(s_D + i, P.D + row);
    }
    cp_async_commit();
  };
  int issued = 0;  // rounds issued (thread 0)
  if (tid == 0) {
    // Dependents may be scheduled as soon as every CTA of this grid is running.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int r = 0; r < L.nbuf && r < nrounds; ++r) {
      issue_round(r);
      issued = r + 1;
    }
  }
  if (nrounds > 0) load_D(0);
  // Everything below reads activations or writes outputs: wait for the grid
  // this launch depends on (returns at once without programmatic dependence).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && c == 0 && L.err != nullptr) *L.err = 0u;

  int cur = -1, qs = 1;  // current problem and its per-token set
  for (int r = 0; r < nrounds; ++r) {
    const int b = r % L.nbuf;
    const uint32_t ph = (uint32_t)(r / L.nbuf) & 1u;
    const int ra = r * RT, re = (ra + RT < nt) ? ra + RT : nt;
    if (r > 0) {
      __syncthreads();  // the previous round's outputs are done with s_D, sq and s_acc
      load_D(r);
    }
    // One segment per problem met in this round.
    for (int sa = ra; sa < re;) {
      if (sa != ra) __syncthreads();  // the previous segment's outputs are done with sq and s_acc
      const int p = problem_of(L, t0 + sa);
      const GemvProblem& P = L.pr[p];
      int se = P.tile0 + P.tiles - t0;
      se = se < re ? se : re;
      const bool newp = p != cur;
      const int K4 = P.K >> 2, total4 = P.M * K4;
      const int G = P.K >> 4, ngroups = P.M * G;
      // One 16-column group per thread, one read of x (staged in shared memory).
      const bool greg = ngroups <= kGemvThreads && ngroups * 64 <= L.xs_bytes;
      if (newp) {
        // Per-token absmax. The other set is cleared for the problem after this one.
        qs ^= 1;
        if (tid < 16) {
          s_amax[(qs ^ 1) * 16 + tid] = 0u;
          s_rs[(qs ^ 1) * 16 + tid] = 0;
        }
        if (greg) {
          // One 16-column group per thread (groups never straddle tokens).
          int m = -1;
          float a = 0.0f;
          if (tid < ngroups) {
            m = tid / G;
            float4 xg[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) xg[j] = load4<kBf16>(P.x, 4 * tid + j);
            a = fmaxf(fmaxf(absmax4(xg[0]), absmax4(xg[1])), fmaxf(absmax4(xg[2]), absmax4(xg[3])));
#pragma unroll
            for (int j = 0; j < 4; ++j) s_xs[4 * tid + j] = xg[j];  // read back after the barrier
          }
          warp_amax(s_amax + qs * 16, m, a);
        } else {
          for (int base = 0; base < total4; base += kXBatch * kGemvThreads) {
            float a[kXBatch];  // all loads of the batch in flight before any reduction
#pragma unroll
            for (int j = 0; j < kXBatch; ++j) {
              const int i4 = base + j * kGemvThreads + tid;
              a[j] = 0.0f;
              if (i4 < total4) a[j] = absmax4(load4<kBf16>(P.x, i4));
            }
#pragma unroll
            for (int j = 0; j < kXBatch; ++j) {
              const int i4 = base + j * kGemvThreads + tid;
              warp_amax(s_amax + qs * 16, i4 < total4 ? i4 / K4 : -1, a[j]);
            }
          }
        }
      }
      for (int i = tid; i < (se - sa) * 16 * 8 * MT; i += kGemvThreads) s_acc[(sa - ra) * 16 * 8 * MT + i] = 0;
      if (newp) {
        __syncthreads();  // absmax complete
        if (greg) {
          int m = -1, sum = 0;
          if (tid < ngroups) {
            m = tid / G;
            const int grp = tid - m * G;
            const float sx = token_scale(s_amax + qs * 16, m);
            // Byte b of word r is column 4b + r of the group: component r of float4 b.
            int q[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 xv = s_xs[4 * tid + j];
              q[j][0] = quant_i8_fast(xv.x, sx);
              q[j][1] = quant_i8_fast(xv.y, sx);
              q[j][2] = quant_i8_fast(xv.z, sx);
              q[j][3] = quant_i8_fast(xv.w, sx);
              sum += q[j][0] + q[j][1] + q[j][2] + q[j][3];
            }
            uint32_t w[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
              w[r] = (uint32_t)(q[0][r] & 0xFF) | ((uint32_t)(q[1][r] & 0xFF) << 8) |
                     ((uint32_t)(q[2][r] & 0xFF) << 16) | ((uint32_t)(q[3][r] & 0xFF) << 24);
            *reinterpret_cast<uint4*>(sq + (int64_t)m * P.q_stride + 16 * grp) = make_uint4(w[0], w[1], w[2], w[3]);
            if (grp == 0) s_sx[qs * 16 + m] = sx;
          }
          warp_rowsum(s_rs + qs * 16, m, sum);
        } else {
          int mprev = -1;
          float sx = 0.0f;
          for (int base = 0; base < total4; base += kXBatch * kGemvThreads) {
            float4 v[kXBatch];
#pragma unroll
            for (int j = 0; j < kXBatch; ++j) {
              const int i4 = base + j * kGemvThreads + tid;
              v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
              if (i4 < total4) v[j] = load4<kBf16>(P.x, i4);
            }
#pragma unroll
            for (int j = 0; j < kXBatch; ++j) {
              const int i4 = base + j * kGemvThreads + tid;
              int m = -1, sum = 0;
              if (i4 < total4) {
                m = i4 / K4;
                const int c4 = i4 - m * K4;
                if (m != mprev) {
                  sx = token_scale(s_amax + qs * 16, m);
                  mprev = m;
                }
                sum = quant_store4(sq, P.q_stride, m, c4, v[j], sx);
                if (c4 == 0) s_sx[qs * 16 + m] = sx;
              }
              warp_rowsum(s_rs + qs * 16, m, sum);
            }
          }
        }
        cur = p;
      }
      __syncthreads();  // codes, scales, row sums and zeroed partial sums visible
      // Tasks of this segment are (tile, 256-code unit) pairs in tile-major
      // order; warp w takes the contiguous range [ntask*w/W, ntask*(w+1)/W), so
      // a warp meets one or two tiles and flushes its sums once per tile.
      const int ntask = (se - sa) * P.n_units;
      const int wpr = P.wpr, nu = P.n_units;
      const bool al = (wpr & 3) == 0;
      // Lane (g, t) reads words 4t..4t+3 of each unit for rows g and g+8, and
      // the activation codes of token g + 8*mt. Lanes past the last token load
      // nothing (their MMA columns are never used), which keeps the shared
      // traffic of the activations to the tokens that exist.
      const uint8_t* qrow[MT];
      bool qon[MT];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        qon[mt] = g + 8 * mt < P.M;
        qrow[mt] = sq + (int64_t)(qon[mt] ? g + 8 * mt : 0) * P.q_stride + 64 * t;
      }
      // One accumulator set per class: four independent MMA chains per unit.
      constexpr int DA = 1;
      int acc[4][DA][MT][4];
      const int tb = (int)(((int64_t)ntask * (warp + 1)) / kGemvWarps);
      int task = (int)(((int64_t)ntask * warp) / kGemvWarps);
      while (task < tb) {
        const int ti = task / nu;
        const int u0 = task - ti * nu;
        const int u1 = (nu < u0 + (tb - task)) ? nu : u0 + (tb - task);
        const int li = sa - ra + ti;  // tile slot in the round buffer
        int okw = 1;
        if (lane == 0) okw = mbar_wait(&full[b * RT + li], ph, abort_flag, L.err, kDevTimeoutProducer) ? 1 : 0;
        okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
        if (!okw) break;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[cc][0][mt][q] = 0;
        const uint32_t* tile = reinterpret_cast<const uint32_t*>(bufs + (size_t)b * L.buf_bytes + s_off[b * RT + li]);
        // Rows past N are not in the tile's slot: lanes on them read nothing.
        const int rv = P.N - (t0 + sa + ti - P.tile0) * 16;
        const bool aon = g < rv, bon = g + 8 < rv;
        const uint32_t* rowa = tile + (aon ? g : 0) * wpr + 4 * t;
        const uint32_t* rowb = tile + (bon ? g + 8 : 0) * wpr + 4 * t;
        for (int u = u0; u < u1; ++u) {
          uint32_t wa[4], wb[4];
          const int w0 = u * 16 + 4 * t;
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
            for (int j = 0; j < 4; ++j) {
              const bool in = w0 + j < wpr;  // words past the row belong to the next row: zero them
              wa[j] = in && aon ? rowa[16 * u + j] : 0u;
              wb[j] = in && bon ? rowb[16 * u + j] : 0u;
            }
          }
          // Half h covers words 2h, 2h+1 of the lane (codes 32h .. 32h+31 of its 64).
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 Q[MT][2];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const uint8_t* qp = qrow[mt] + 256 * u + 32 * h;
              Q[mt][0] = make_uint4(0u, 0u, 0u, 0u);
              Q[mt][1] = make_uint4(0u, 0u, 0u, 0u);
              if (qon[mt]) {
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
                const uint4& q0 = Q[mt][0];
                const uint4& q1 = Q[mt][1];
                const uint32_t b0 = cc == 0 ? q0.x : (cc == 1 ? q0.y : (cc == 2 ? q0.z : q0.w));
                const uint32_t b1 = cc == 0 ? q1.x : (cc == 1 ? q1.y : (cc == 2 ? q1.z : q1.w));
                mma_u8s8(acc[cc][0][mt], a0, a1, a2, a3, b0, b1);
              }
            }
          }
        }
        flush_tile<MT, DA>(acc, s_acc + (size_t)li * 16 * 8 * MT, g, t);
        task += u1 - u0;
      }
      cp_async_wait_all();  // this thread's row-scale copies
      __syncthreads();
      if (*abort_flag) {
        // Block-uniform after the barrier. Let the copies already issued land
        // before the CTA exits.
        if (tid == 0) {
          for (int rr = r; rr < issued; ++rr) {
            const int bb = rr % L.nbuf, na = (rr * RT + RT < nt ? RT : nt - rr * RT);
            for (int li = 0; li < na; ++li)
              mbar_wait(&full[bb * RT + li], (uint32_t)(rr / L.nbuf) & 1u, nullptr, L.err, kDevTimeoutDrain,
                        100000000ull);
          }
        }
        return;
      }
      // This round's buffer is consumed once its last segment is: start the
      // round that reuses it while the outputs are written.
      if (se == re && tid == 0 && r + L.nbuf < nrounds) {
        issue_round(r + L.nbuf);
        issued = r + L.nbuf + 1;
      }
      // Outputs of this segment: rows x tokens, coalesced along the rows.
      const int nout = (se - sa) * 16 * P.M;
      for (int idx = tid; idx < nout; idx += kGemvThreads) {
        const int tok = idx / ((se - sa) * 16);
        const int rr = idx - tok * (se - sa) * 16;
        const int ti2 = rr >> 4, r16 = rr & 15;
        const int64_t row = (int64_t)(t0 + sa + ti2 - P.tile0) * 16 + r16;
        if (row >= P.N) continue;
        const int a = s_acc[((size_t)(sa - ra + ti2) * 16 + r16) * 8 * MT + tok] - s_rs[qs * 16 + tok];
        if (kAccOut)
          P.acc[(int64_t)tok * P.N + row] = a;
        else
          P.y[(int64_t)tok * P.N + row] = rescale(a, s_sx[qs * 16 + tok], s_D[(sa - ra + ti2) * 16 + r16]);
      }
      sa = se;
    }
  }
}

template <int MT, bool kAccOut, bool kBf16>
static cudaError_t launch_gemv_t(const GemvLaunch& L, int grid, size_t smem, bool pdl, cudaStream_t stream) {
  auto kern = gemv_kernel<MT, kAccOut, kBf16>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, L);
}

static size_t gemv_smem_bytes(const GemvLaunch& L, int MT) {
  return (size_t)L.nbuf * L.buf_bytes + L.q_bytes + L.xs_bytes + 3 * 32 * 4 + (size_t)L.round_tiles * 16 * 4 +
         (size_t)L.round_tiles * 16 * 8 * MT * 4 + (size_t)L.nbuf * L.round_tiles * (8 + 4) + 16;
}

// Shared-memory bytes of launch tile gt (rows x K/4 rounded up to 128 B).
static int64_t host_tile_bytes(const GemvLaunch& L, int gt) {
  int p = 0;
  while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
  const GemvProblem& P = L.pr[p];
  const int64_t row0 = (int64_t)(gt - P.tile0) * 16;
  const int64_t rows = P.N - row0 < 16 ? P.N - row0 : 16;
  return (rows * P.wpr * 4 + 127) / 128 * 128;
}

// Split the launch's tiles into `grid` contiguous ranges of about equal bytes
// (problems of different K have tiles of different size). Returns the largest
// range in bytes and the largest range in tiles.
static void partition_by_bytes(GemvLaunch& L, int grid, int64_t* max_bytes, int* max_tiles) {
  int64_t total = 0;
  for (int gt = 0; gt < L.total_tiles; ++gt) total += host_tile_bytes(L, gt);
  int64_t acc = 0, best_b = 0, cur_b = 0;
  int c = 0, best_t = 0, start = 0;
  L.cta_start[0] = 0;
  for (int gt = 0; gt < L.total_tiles; ++gt) {
    const int64_t tb = host_tile_bytes(L, gt);
    // Close CTA c once it holds its share, keeping at least one tile for each later CTA.
    const int64_t target = total * (c + 1) / grid;
    if (c + 1 < grid && gt > start && acc + tb / 2 > target && L.total_tiles - gt >= grid - c - 1) {
      best_b = cur_b > best_b ? cur_b : best_b;
      best_t = gt - start > best_t ? gt - start : best_t;
      L.cta_start[++c] = gt;
      start = gt;
      cur_b = 0;
    }
    acc += tb;
    cur_b += tb;
  }
  best_b = cur_b > best_b ? cur_b : best_b;
  best_t = L.total_tiles - start > best_t ? L.total_tiles - start : best_t;
  // Any CTA left without tiles gets an empty range.
  for (int k = c + 1; k <= grid; ++k) L.cta_start[k] = L.total_tiles;
  *max_bytes = best_b;
  *max_tiles = best_t;
}

int64_t gemv_stage_bytes(int64_t K) { return ((16 * (K / 4)) + 127) / 128 * 128; }

bool gemv_group_fits(int64_t maxM, int64_t maxK) {
  if (maxM > kGemvMaxM) return false;
  const int64_t q = (maxM * gemv_q_stride(maxK) + 127) / 128 * 128;
  const int64_t xs = maxM * maxK <= 16 * kGemvThreads ? maxM * maxK * 4 : 0;
  return q + xs + 2 * gemv_stage_bytes(maxK) + 16 * 1024 <= kGemvMaxSmem;
}

cudaError_t launch_gemv_group(const GemvCall* calls, int n, uint32_t* err, bool pdl, cudaStream_t stream,
                              int num_sms) {
  if (n < 1 || n > kGemvMaxGroup) return cudaErrorInvalidValue;
  GemvLaunch L;
  std::memset(&L, 0, sizeof(L));
  int64_t maxM = 0, maxK = 0;
  int tiles = 0;
  for (int i = 0; i < n; ++i) {
    GemvProblem& P = L.pr[i];
    P.x = calls[i].x;
    P.packed = calls[i].packed;
    P.D = calls[i].D;
    P.y = calls[i].y;
    P.acc = calls[i].acc;
    P.M = (int)calls[i].M;
    P.N = (int)calls[i].N;
    P.K = (int)calls[i].K;
    P.wpr = P.K / 16;
    P.n_units = (P.wpr + 15) / 16;
    P.tiles = (P.N + 15) / 16;
    P.tile0 = tiles;
    P.q_stride = (int)gemv_q_stride(P.K);
    tiles += P.tiles;
    maxM = calls[i].M > maxM ? calls[i].M : maxM;
    maxK = calls[i].K > maxK ? calls[i].K : maxK;
  }
  L.nprob = n;
  L.total_tiles = tiles;
  L.err = err;
  L.stage_bytes = (int)gemv_stage_bytes(maxK);
  L.q_bytes = (int)((maxM * gemv_q_stride(maxK) + 127) / 128 * 128);
  // Problems with at most one 16-column group per thread stage x in shared memory.
  int64_t xs = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t mk = calls[i].M * calls[i].K;
    if (mk / 16 <= kGemvThreads && mk * 4 > xs) xs = mk * 4;
  }
  L.xs_bytes = (int)xs;
  const int MT = maxM <= 8 ? 1 : 2;
  int grid0 = tiles < num_sms ? tiles : num_sms;
  if (grid0 > kGemvMaxGrid) grid0 = kGemvMaxGrid;
  int64_t cta_bytes = 0;
  int per_cta = 0;
  partition_by_bytes(L, grid0, &cta_bytes, &per_cta);
  // Per tile slot: its partial-sum block, row scales, barrier and offset entry.
  const int64_t slot_extra = 16 * 8 * MT * 4 + 16 * 4 + 8 + 4;
  const int64_t fixed = L.q_bytes + L.xs_bytes + 3 * 32 * 4 + 16;
  if (fixed + cta_bytes + per_cta * slot_extra <= kGemvMaxSmem) {
    L.nbuf = 1;  // every tile of a CTA in flight at once
    L.round_tiles = per_cta;
    L.buf_bytes = (int)cta_bytes;
  } else {
    L.nbuf = 2;
    int64_t rt = (kGemvSmemTarget - fixed) / (2 * (L.stage_bytes + slot_extra));
    if (rt < 1) rt = 1;
    L.round_tiles = (int)rt;
    L.buf_bytes = (int)(rt * L.stage_bytes);
  }
  const size_t smem = gemv_smem_bytes(L, MT);
  if ((int64_t)smem > kGemvMaxSmem) return cudaErrorInvalidValue;
  const int grid = grid0;
  const bool accout = calls[0].acc != nullptr;
  const bool bf16 = calls[0].bf16;
  for (int i = 1; i < n; ++i)
    if (calls[i].bf16 != bf16) return cudaErrorInvalidValue;  // one input type per launch
#define BL_GEMV(MTV, AO, BF) \
  if (MT == MTV && accout == AO && bf16 == BF) return launch_gemv_t<MTV, AO, BF>(L, grid, smem, pdl, stream);
  BL_GEMV(1, false, false)
  BL_GEMV(1, true, false)
  BL_GEMV(2, false, false)
  BL_GEMV(2, true, false)
  BL_GEMV(1, false, true)
  BL_GEMV(1, true, true)
  BL_GEMV(2, false, true)
  BL_GEMV(2, true, true)
#undef BL_GEMV
  return cudaErrorInvalidValue;
}

}  // namespace bl
