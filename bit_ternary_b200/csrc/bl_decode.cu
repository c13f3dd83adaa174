// bl_decode.cu - decode BitLinear (M <= 16 tokens) for one or several
// independent BitLinears per launch: ActQuant (or RMSNorm + ActQuant) of the
// activations inside every CTA, the packed ternary weights streamed once from
// HBM through per-warp shared-memory stages, an exact int32 contraction and
// the fp32 rescale in the epilogue.
//
// The operation is the BitLinear product of "Core AI model zoo - BitVLA",
// section 2 (M=1 decode, arbitrary K with K % 16 == 0, any N, per-row scale
// D [N,1]), with the wrapper's ActQuant (section 1) done inside the kernel.
//
// Streaming. The packed weights are the only large stream (2 bits per weight).
// Work is cut into tiles of 16 consecutive rows, and a tile into tasks: the
// whole tile when every warp of a CTA gets two or more tiles, else chunks of
// units so that all warps share a short launch (chunk j of tile i is one
// task). Every CTA owns a contiguous, byte-balanced range of tiles over all
// problems of the launch; its 8 warps take every 8th task in (tile, chunk)
// order, and walk each task in groups of up to 4 256-code units. A warp
// copies each group (16 rows x 256 bytes) with 16-byte cp.async into one of
// its two shared-memory stages, each copy instruction covering whole
// 128-byte lines, and contracts one stage while the next group lands; it
// waits only on its own copies (cp.async.wait_group + __syncwarp). The copies
// carry an L2 evict-first policy: the weights are read once. The first group
// of every warp is issued before griddepcontrol.wait (weights never depend on
// the previous kernel), so under programmatic dependent launch a launch's
// weights stream while the previous launch still runs; without that
// dependency the activations are loaded first, ahead of the weight stream.
// (One bulk-copy engine per SM moves only about 20-25 GB/s, far below a
// B200 SM's share of HBM bandwidth, so the stream goes through the load/store
// units of all warps instead.)
//
// Accumulation. A chunk's partial sums go to its tile's block in shared
// memory (one of 16 slots, by tile index) with shared atomics: exact integers,
// so the order does not matter. The warp that adds the tile's last chunk
// writes the outputs, clears the block and hands the slot to tile i + 16. A
// warp that holds a whole tile writes its outputs directly from registers.
//
// Math. Lane (g, t) = (lane/4, lane%4) holds words 4t..4t+3 of each unit for
// rows g and g+8 of the tile. For class c in 0..3, word & (0x03030303 << 2c)
// leaves in byte b the value (code[4b+c]+1) << 2c: one AND gives four u8
// operands of mma.sync.m16n8k32 (u8 weights x s8 activations). One accumulator
// set per class, recombined exactly as acc0 + acc1/4 + acc2/16 + acc3/64, gives
// sum q*(code+1); subtracting sum q gives the signed result.
//
// Activations in shared memory. A token's codes are stored per 256-code unit.
// Word w = 4t + 2h + j of a unit (codes 16w..16w+15) splits into four class
// words: class c holds the codes of columns {c, 4+c, 8+c, 12+c}, the order in
// which a masked weight word presents them. Inside the 32-byte chunk
// 128h + 32t, class c of word j sits at 8c + 4j, so one 16-byte load gives the
// B operands (words 2h and 2h+1) of two classes as aligned register pairs.
// Lane (g, t) reads its 32 bytes of half h at 128h + 32t: the four lanes of a
// token cover 128 distinct bytes, and the row stride of 16 (mod 128) bytes
// moves the next token onto the other banks.
#include "bl_internal.h"

#include <atomic>
#include <cstring>
#include <utility>

namespace bl {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecMaxGrid = 3 * 160;
constexpr int kDecRegGroups = 2;  // 16-column groups per thread held in registers by the quantiser
constexpr int kDecTok = kDecodeMaxGroup * 16;  // per-token state entries: problem * 16 + token

// Units per task (the register buffer of one task): eight 32-bit registers
// per unit, two tasks in flight.
template <int MT>
__host__ __device__ constexpr int dec_upt() { return 4; }
// Pipeline stages per warp (S - 1 groups of copies in flight).
constexpr int kDecStages = 2;

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

// The launch's problems and common arguments.
struct DecHead {
  DecProblem pr[kDecodeMaxGroup];
  const float* g;  // RMSNorm mode: norm weight [K] (one problem per launch)
  float eps;
  int nprob;
  int total_tiles;
  int q_bytes;
  int pdl;       // launched as a programmatic dependent of the previous work in the stream
  int acc_cols;  // token columns of a slot's partial-sum block: the largest M
  uint32_t* err;
};

struct DecLaunch {
  DecHead h;
  int cta_start[kDecMaxGrid + 1];  // CTA c owns launch tiles [cta_start[c], cta_start[c+1])
};

// Shared memory past the activation codes.
__host__ __device__ constexpr int dec_fixed_bytes(int acc_cols, int S) {
  return 0
         + kDecodeSlots * 16 * acc_cols * 4  // s_acc
         + kDecodeSlots * 16 * 4         // s_D
         + 3 * kDecTok * 4               // s_sx, s_rs, s_amax
         + 2 * kDecodeSlots * 4          // s_cnt, s_gen
         + 16 * (8 + 4 + 4)              // RMSNorm: sums of squares, mean squares, flags
         + 64;                           // abort flag
}

__device__ __forceinline__ void dec_mma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte load of streamed weights: read once, not kept in L1.
__device__ __forceinline__ uint4 ldg_stream(const uint32_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
}

// Barrier of the CTA's 8 warps (named, so that its count is explicit).
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kDecThreads) : "memory"); }

__device__ __forceinline__ int dec_problem_of(const DecHead& L, int gt) {
  int p = 0;
#pragma unroll 1
  while (p + 1 < L.nprob && gt >= L.pr[p + 1].tile0) ++p;
  return p;
}

// Byte offset, inside a unit, of the codes of word w = 4t + 2h + j (see the
// file header): the 32-byte chunk 128h + 32t, where class c of word j (its
// 4 codes for columns {c, 4+c, 8+c, 12+c}) sits at 8c + 4j.
__device__ __forceinline__ int dec_group_slot(int w) { return 128 * ((w >> 1) & 1) + 32 * (w >> 2) + 4 * (w & 1); }

// Shared-memory address of the codes of group gi (columns 16gi..16gi+15) of
// token m; its class c word goes to this address + 8c.
__device__ __forceinline__ uint8_t* dec_q_group(uint8_t* sq, const DecProblem& P, int m, int gi) {
  return sq + P.q_off + m * P.q_stride + 256 * (gi >> 4) + dec_group_slot(gi & 15);
}

// Store a group's four class words (w[c]: the codes of columns {c, 4+c, 8+c,
// 12+c}) at dec_q_group's address.
__device__ __forceinline__ void dec_store_group(uint8_t* dst, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  *reinterpret_cast<uint32_t*>(dst) = w0;
  *reinterpret_cast<uint32_t*>(dst + 8) = w1;
  *reinterpret_cast<uint32_t*>(dst + 16) = w2;
  *reinterpret_cast<uint32_t*>(dst + 24) = w3;
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
  dec_store_group(dst, w[0], w[1], w[2], w[3]);
  return sum;
}

// What the contraction of a group in flight needs, packed in four words (the
// same for every lane): the activation offset of its first unit (token 0),
// the tile's CTA-local index, and
// problem | chunk << 3 | units << 20 | first << 24 | last << 25 | valid << 26.
struct __align__(16) DecRun {
  int qoff, i, meta, pad;
  __device__ __forceinline__ int p() const { return meta & 7; }
  __device__ __forceinline__ int j() const { return (meta >> 3) & 0x1FFFF; }
  __device__ __forceinline__ int n() const { return (meta >> 20) & 15; }
  __device__ __forceinline__ bool first() const { return (meta >> 24) & 1; }
  __device__ __forceinline__ bool last() const { return (meta >> 25) & 1; }
  __device__ __forceinline__ bool valid() const { return (meta >> 26) & 1; }
};

// Asynchronous copies of 16 or 4 bytes global -> shared. With src_bytes == 0
// the destination is zero-filled; the source address must still lie inside
// an allocation (callers pass the buffer's first element).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
               "l"(__cvta_generic_to_global(src)), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(__cvta_generic_to_global(src))
               : "memory");
}
// The same with an L2 cache policy (the streamed weights are read once).
__device__ __forceinline__ void cp_async16_zfill_pol(void* dst, const void* src, uint32_t src_bytes, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_u32(dst)),
               "l"(__cvta_generic_to_global(src)), "r"(src_bytes), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async16_pol(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
               "l"(__cvta_generic_to_global(src)), "l"(pol)
               : "memory");
}
// As cp_async16_pol, with the destination given as a 32-bit shared address
// plus a compile-time offset (folded into the instruction).
template <int OFF>
__device__ __forceinline__ void cp_async16_pol_at(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0+%3], [%1], 16, %2;" ::"r"(dst),
               "l"(__cvta_generic_to_global(src)), "l"(pol), "n"(OFF)
               : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void cp_async4_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)),
               "l"(__cvta_generic_to_global(src)), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The fast path's copies: copy m goes to d0 + m * ROWB (a compile-time offset)
// from s0 + m * rstep words.
template <int ROWB, int... Ms>
__device__ __forceinline__ void dec_fast_copies(uint32_t d0, const uint32_t* s0, int64_t rstep, uint64_t pol,
                                                std::integer_sequence<int, Ms...>) {
  (cp_async16_pol_at<Ms * ROWB>(d0, s0 + Ms * rstep, pol), ...);
}

// One pipeline stage of a warp holds a group's 16 rows, UPT * 64 bytes each
// and unpadded, then two row scales per lane. Lanes (g, t) and (g + 1, t) read
// in the same quarter-warp, so rows g and g + 1 must use different halves of
// the 128-byte bank window: with an even UPT (row stride 0 mod 128) the
// 64-byte halves of every odd row are swapped (16-byte chunk c is stored at
// position c ^ 4); with an odd UPT the stride alone offsets them.
template <int UPT>
__host__ __device__ constexpr int dec_row_stride() { return UPT * 64; }
template <int UPT>
__host__ __device__ constexpr int dec_stage_bytes() { return 16 * dec_row_stride<UPT>() + 256; }
template <int UPT>
__device__ __forceinline__ int dec_chunk_pos(int row, int chunk) {
  return (UPT & 1) ? chunk : chunk ^ (4 * (row & 1));
}

// A warp's position in its work: tasks warp, warp + 8, warp + 16, ... in
// (tile, chunk) order (chunk j of the CTA's tile i, in problem p), each task
// cut into groups of at most UPT units. The current problem's fields are kept
// in registers, so stepping reads the launch parameters only when the
// problem changes.
template <int UPT, bool kAccOut>
struct DecCursor {
  // task position
  int p, C, i, j, pend;
  bool valid;
  // the current problem
  const uint32_t* packed;
  const float* D;
  int wpr, N, tile0, upt, nu, q_off;
  // the current task
  const uint32_t* src;  // the lane's first copy source: row lane / CPR, chunk lane % CPR of unit u
  int w0;               // word of that chunk in its row: 16*u + 4*(lane % CPR)
  int left;             // units of the task not yet issued
  uint64_t pol;         // L2 policy of the weight copies: evict first
  int qoff;             // activation offset of unit u (token 0)
  int row0, rv;
  bool first;

  __device__ __forceinline__ void load_problem(const DecHead& L, int t0) {
    const DecProblem& P = L.pr[p];
    packed = P.packed;
    D = P.D;
    wpr = P.wpr;
    N = P.N;
    tile0 = P.tile0;
    upt = P.upt;
    nu = P.nu;
    q_off = P.q_off;
    C = P.nchunk;
    pend = P.tile0 + P.tiles - t0;
  }
  // Move (i, j) onto a task: whole tiles are skipped at once, one problem at
  // a time.
  __device__ __forceinline__ void normalise(const DecHead& L, int t0, int nt) {
    while (j >= C && i < nt) {
      const int adv = C == 1 ? j : j / C;
      if (i + adv < pend) {
        i += adv;
        j -= adv * C;
      } else {
        j -= (pend - i) * C;
        i = pend;
        if (i < nt && p + 1 < L.nprob) {
          ++p;
          load_problem(L, t0);
        }
      }
    }
  }
  // Set up the task at (i, j).
  // Copies: a group's 16 rows x (4 * UPT) 16-byte chunks are spread over the
  // lanes so that one copy instruction covers whole rows (full 128-byte
  // lines): chunk lane + 32m is row m * RPM + lane / CPR, chunk lane % CPR.
  static constexpr int CPR = 4 * UPT;  // chunks per row
  static constexpr int RPM = 32 / CPR;  // rows per copy instruction
  static_assert(32 % CPR == 0 && 16 % RPM == 0, "a copy instruction covers whole rows");
  __device__ __forceinline__ void open(int t0, int nt, int lane) {
    valid = i < nt;
    if (!valid) return;
    row0 = (t0 + i - tile0) * 16;
    rv = N - row0 < 16 ? N - row0 : 16;
    const int ua = j * upt;
    const int ue = ua + upt < nu ? ua + upt : nu;
    w0 = 16 * ua + 4 * (lane % CPR);
    src = packed + (int64_t)(row0 + lane / CPR) * wpr + w0;
    qoff = q_off + 256 * ua;
    left = ue - ua;
    first = true;
  }
  __device__ __forceinline__ void init(const DecHead& L, int t0, int nt, int warp, int lane) {
    p = dec_problem_of(L, t0);
    load_problem(L, t0);
    pol = l2_policy_evict_first();
    i = 0;
    j = warp;
    normalise(L, t0, nt);
    open(t0, nt, lane);
  }
  // Start the copies of the next group into `stage` and return what its
  // contraction needs (valid() == false past the warp's last task; nothing
  // is copied then, but the caller still commits a copy group). Rows past N
  // and words past the row (or past the group's units) are zero-filled. A
  // group that opens its task also brings row scales: D[row0 + lane] (lanes
  // 0..15, chunked tiles) or D[row0 + g] and D[row0 + g + 8] (whole tiles).
  // The copies land only for this lane: the warp synchronises before reading.
  __device__ __forceinline__ DecRun issue(const DecHead& L, int t0, int nt, uint8_t* stage, int lane) {
    DecRun r;
    r.pad = 0;
    if (!valid) {
      r.qoff = r.i = r.meta = 0;
      return r;
    }
    constexpr int RS = dec_row_stride<UPT>();
    const int n = left < UPT ? left : UPT;
    const int lr = lane / CPR, lc = lane % CPR;
    // destination of the lane's chunk in row m * RPM + lr
    auto dst = [&](int m) { return stage + (m * RPM + lr) * RS + 16 * dec_chunk_pos<UPT>(m * RPM + lr, lc); };
    const int64_t rstep = (int64_t)RPM * wpr;  // words between a lane's rows
    if (rv == 16 && n == UPT && (wpr & 3) == 0 && w0 - 4 * lc + 16 * UPT <= wpr) {
      // Every row present and every unit whole. With an even number of rows
      // per copy instruction every row of this lane has the parity of lr, so
      // the destinations are one base plus constant offsets.
      if constexpr (RPM % 2 == 0 || (UPT & 1)) {
        const uint32_t d0 = smem_u32(dst(0));
        const uint32_t* s0 = src;
        dec_fast_copies<RPM * RS>(d0, s0, rstep, pol, std::make_integer_sequence<int, 16 / RPM>{});
      } else {
#pragma unroll
        for (int m = 0; m < 16 / RPM; ++m) cp_async16_pol(dst(m), src + m * rstep, pol);
      }
    } else if ((wpr & 3) == 0) {
      // Rows start 16-byte aligned; a chunk is wholly in the row or past it.
#pragma unroll
      for (int m = 0; m < 16 / RPM; ++m) {
        const bool in = m * RPM + lr < rv && lc < 4 * n && w0 < wpr;
        cp_async16_zfill_pol(dst(m), in ? src + m * rstep : packed, in ? 16u : 0u, pol);
      }
    } else {
      // Rows not 16-byte aligned: 4-byte copies.
#pragma unroll
      for (int m = 0; m < 16 / RPM; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = m * RPM + lr < rv && lc < 4 * n && w0 + e < wpr;
          cp_async4_zfill(dst(m) + 4 * e, in ? src + m * rstep + e : packed, in ? 4u : 0u);
        }
    }
    if (!kAccOut && first) {
      const int g = lane >> 2;
      float* dd = reinterpret_cast<float*>(stage + 16 * RS) + 2 * lane;
      if (C > 1) {
        const bool in = j == 0 && lane < 16 && row0 + lane < N;
        cp_async4_zfill(dd, in ? D + row0 + lane : D, in ? 4u : 0u);
      } else {
        cp_async4_zfill(dd, g < rv ? D + row0 + g : D, g < rv ? 4u : 0u);
        cp_async4_zfill(dd + 1, g + 8 < rv ? D + row0 + g + 8 : D, g + 8 < rv ? 4u : 0u);
      }
    }
    const bool last = left == n;
    r.qoff = qoff;
    r.i = i;
    r.meta = p | ((j & 0x1FFFF) << 3) | (n << 20) | ((int)first << 24) | ((int)last << 25) | (1 << 26);
    if (last) {
      j += kDecWarps;
      normalise(L, t0, nt);
      open(t0, nt, lane);
    } else {
      left -= n;
      first = false;
      src += 16 * n;
      w0 += 16 * n;
      qoff += 256 * n;
    }
    return r;
  }
};

// Problems [pa, pb] of this CTA, flattened into 16-column groups: group gg
// belongs to problem p with pre[p - pa] <= gg < pre[p - pa + 1].
struct DecGroups {
  int pa, np, total;
  int pre[kDecodeMaxGroup + 1];
  __device__ __forceinline__ void locate(const DecHead& L, int gg, int& p, int& m, int& gi) const {
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
  for (int j = 0; j < 4; ++j) f[j] = load4_dep<kX == kDecBf16>(P.x, i4 + j);
}

// ActQuant of every token of the CTA's problems into shared memory (fp32 or
// bf16 activations), in two parts. dec_quant_load reads the first
// kDecRegGroups 16-column groups of each thread into registers (a launch
// without a dependency issues it before any weight copy, so that these loads
// do not queue behind the weight stream); dec_quant_rest finishes: per-token
// max|x| by shared atomics, then the codes, s_x and the row sums.
// Groups beyond the registers are read twice (for the maximum, then for the
// codes), two at a time so that their loads are in flight together. Run by
// the 256 consumer threads.
template <int kX>
__device__ __forceinline__ void dec_quant_load(const DecHead& L, const DecGroups& G, float4 (&f)[kDecRegGroups][4]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) {
    const int gg = tid + r * kDecThreads;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      dec_load_group<kX>(L.pr[p], m, gi, f[r]);
    }
  }
}

template <int kX>
__device__ void dec_quant_rest(const DecHead& L, const DecGroups& G, float4 (&f)[kDecRegGroups][4], uint8_t* sq,
                               float* s_sx, int32_t* s_rs, uint32_t* s_amax) {
  const int tid = threadIdx.x;
  constexpr int B = 2;  // groups beyond the registers loaded together
  auto absmax16 = [](const float4 (&v)[4]) {
    return fmaxf(fmaxf(dec_absmax4(v[0]), dec_absmax4(v[1])), fmaxf(dec_absmax4(v[2]), dec_absmax4(v[3])));
  };
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) {
    const int gg = tid + r * kDecThreads;
    int tok = -1;
    float a = 0.0f;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      tok = p * 16 + m;
      a = absmax16(f[r]);
    }
    dec_amax(s_amax, tok, a);
  }
  for (int base = kDecRegGroups * kDecThreads; base < G.total; base += B * kDecThreads) {
    float4 v[B][4];
    int tok[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int gg = base + b * kDecThreads + tid;
      tok[b] = -1;
      if (gg < G.total) {
        int p, m, gi;
        G.locate(L, gg, p, m, gi);
        dec_load_group<kX>(L.pr[p], m, gi, v[b]);
        tok[b] = p * 16 + m;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) dec_amax(s_amax, tok[b], tok[b] >= 0 ? absmax16(v[b]) : 0.0f);
  }
  consumers_sync();  // every token's max|x| is complete
  auto codes = [&](const float4 (&v)[4], int gg) {
    int tok = -1, sum = 0;
    if (gg < G.total) {
      int p, m, gi;
      G.locate(L, gg, p, m, gi);
      tok = p * 16 + m;
      const float sx = __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[tok]), kFloor));
      sum = dec_quant_group(v, sx, dec_q_group(sq, L.pr[p], m, gi));
      if (gi == 0) s_sx[tok] = sx;
    }
    dec_rowsum(s_rs, tok, sum);
  };
#pragma unroll
  for (int r = 0; r < kDecRegGroups; ++r) codes(f[r], tid + r * kDecThreads);
  for (int base = kDecRegGroups * kDecThreads; base < G.total; base += B * kDecThreads) {
    float4 v[B][4];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int gg = base + b * kDecThreads + tid;
      if (gg < G.total) {
        int p, m, gi;
        G.locate(L, gg, p, m, gi);
        dec_load_group<kX>(L.pr[p], m, gi, v[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) codes(v[b], base + b * kDecThreads + tid);
  }
}

// Prepared activations (int8 codes already in the private order, natural
// group order, row stride K; s_x and row sums): copied into the shared layout.
__device__ void dec_load_prepared(const DecHead& L, const DecGroups& G, uint8_t* sq, float* s_sx, int32_t* s_rs) {
  const int tid = threadIdx.x;
  constexpr int B = 4;  // groups per thread whose loads are in flight together
  for (int base = 0; base < G.total; base += B * kDecThreads) {
    uint4 v[B];
    uint8_t* dst[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int gg = base + b * kDecThreads + tid;
      dst[b] = nullptr;
      if (gg < G.total) {
        int p, m, gi;
        G.locate(L, gg, p, m, gi);
        const DecProblem& P = L.pr[p];
        v[b] = reinterpret_cast<const uint4*>(static_cast<const int8_t*>(P.x) + (int64_t)m * P.K)[gi];
        dst[b] = dec_q_group(sq, P, m, gi);
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b)
      if (dst[b] != nullptr) dec_store_group(dst[b], v[b].x, v[b].y, v[b].z, v[b].w);
  }
  for (int i = tid; i < G.np * 16; i += kDecThreads) {
    const int p = G.pa + (i >> 4), m = i & 15;
    if (m < L.pr[p].M) {
      s_sx[p * 16 + m] = L.pr[p].sx_in[m];  // plain loads: written by the grid waited for
      s_rs[p * 16 + m] = L.pr[p].rs_in[m];
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
__device__ void dec_rms_quantise(const DecHead& L, const DecGroups& G, uint8_t* sq, float* s_sx, int32_t* s_rs,
                                 uint32_t* s_amax, double* s_ss, float* s_ms, int* s_flag,
                                 unsigned long long* bins) {
  const int tid = threadIdx.x;
  const DecProblem& P = L.pr[0];
  const int Gk = P.K >> 4;
  const float4* g4 = reinterpret_cast<const float4*>(L.g);
  float4 f[kDecRegGroups][4];
  // Sum of squares per token.
  for (int base = 0; base < G.total; base += kDecThreads) {
    const int r = base / kDecThreads;
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
    for (int b = tid; b < kRmsBins; b += kDecThreads) bins[b] = 0ull;
    consumers_sync();
    const float4* xr = reinterpret_cast<const float4*>(P.x) + ((int64_t)m * P.K >> 2);
    for (int i4 = tid; i4 < (P.K >> 2); i4 += kDecThreads) {
      const float4 v = xr[i4];  // x may come from the grid waited for: no read-only path
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
  for (int base = 0; base < G.total; base += kDecThreads) {
    const int r = base / kDecThreads;
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
  for (int base = 0; base < G.total; base += kDecThreads) {
    const int r = base / kDecThreads;
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
__global__ void __launch_bounds__(kDecThreads, MT == 1 ? 2 : 1) bl_ternary_decode_kernel(const __grid_constant__ DecLaunch LP) {
  constexpr int UPT = dec_upt<MT>();
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;                                                      // [warp][stage]
  constexpr int S = kDecStages;
  uint8_t* sq = smem + kDecWarps * S * dec_stage_bytes<UPT>();
  int32_t* s_acc = reinterpret_cast<int32_t*>(sq + LP.h.q_bytes);             // [slot][16 rows][acc_cols tokens]
  const int AC = LP.h.acc_cols;
  float* s_D = reinterpret_cast<float*>(s_acc + kDecodeSlots * 16 * AC);      // [slot][16]
  float* s_sx = s_D + kDecodeSlots * 16;                                       // [problem * 16 + token]
  int32_t* s_rs = reinterpret_cast<int32_t*>(s_sx + kDecTok);
  uint32_t* s_amax = reinterpret_cast<uint32_t*>(s_rs + kDecTok);
  int32_t* s_cnt = reinterpret_cast<int32_t*>(s_amax + kDecTok);  // chunks added per slot
  int32_t* s_gen = s_cnt + kDecodeSlots;                           // slot s holds tile s + 16 * s_gen[s]
  double* s_ss = reinterpret_cast<double*>(s_gen + kDecodeSlots);  // RMSNorm: [16] sums of squares
  float* s_ms = reinterpret_cast<float*>(s_ss + 16);               // [16] mean squares
  int* s_flag = reinterpret_cast<int*>(s_ms + 16);                 // [16] exact path needed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(s_flag + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;

  // Dependents may be scheduled as soon as every CTA of this grid is running.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const DecHead& L = LP.h;
  const int t0 = LP.cta_start[c];
  const int nt = LP.cta_start[c + 1] - t0;
  if (nt <= 0) return;

  DecGroups G;
  G.pa = dec_problem_of(L, t0);
  G.np = dec_problem_of(L, t0 + nt - 1) - G.pa + 1;
  G.pre[0] = 0;
#pragma unroll
  for (int i = 0; i < kDecodeMaxGroup; ++i)
    G.pre[i + 1] = G.pre[i] + (i < G.np ? L.pr[G.pa + i].M * (L.pr[G.pa + i].K >> 4) : 0);
  G.total = G.pre[kDecodeMaxGroup];

  // Without a programmatic dependency nothing this launch reads is still
  // being written, and the activations' loads go first, ahead of the weight
  // stream in the memory queues.
  constexpr bool kRegQuant = kX == kDecF32 || kX == kDecBf16;
  const bool early_x = kRegQuant && !L.pdl;
  float4 f[kDecRegGroups][4];
  if (early_x) dec_quant_load<kX>(L, G, f);

  // The first groups' weights (one per stage) are requested at once: they
  // never depend on the grid this launch waits for.
  constexpr int SB = dec_stage_bytes<UPT>();
  constexpr int RS = dec_row_stride<UPT>();
  uint8_t* wstage = stages + (size_t)warp * S * SB;  // this warp's S stages
  DecCursor<UPT, kAccOut> cur;
  cur.init(L, t0, nt, warp, lane);
  // What each stage's contraction needs, in registers (two stages: the
  // stage index selects one of two records).
  static_assert(S == 2, "one register record per stage");
  DecRun rec0 = cur.issue(L, t0, nt, wstage, lane);
  cp_async_commit();
  DecRun rec1 = cur.issue(L, t0, nt, wstage + SB, lane);
  cp_async_commit();

  for (int i = tid; i < kDecodeSlots * 16 * AC; i += kDecThreads) s_acc[i] = 0;
  if (tid < kDecodeSlots) {
    s_cnt[tid] = 0;
    s_gen[tid] = 0;
  }
  if (tid < kDecTok) {
    s_amax[tid] = 0u;
    s_rs[tid] = 0;
  }
  if (tid < 16) s_ss[tid] = 0.0;
  if (tid == 0) *abort_flag = 0;

  // The activations may be written by the grid this launch depends on: only
  // an L2 prefetch (no data is consumed) before the dependency wait.
  if (!early_x) {
    const int esz = kX == kDecBf16 ? 2 : (kX == kDecPrepared ? 1 : 4);
    for (int i = 0; i < G.np; ++i) {
      const DecProblem& P = L.pr[G.pa + i];
      const int64_t bytes = (int64_t)P.M * P.K * esz;
      for (int64_t o = (int64_t)tid * 128; o < bytes; o += (int64_t)kDecThreads * 128)
        prefetch_l2(static_cast<const uint8_t*>(P.x) + o);
    }
  }
  consumers_sync();  // shared state initialised (before the wait, where it costs nothing)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && c == 0 && L.err != nullptr) *L.err = 0u;

  if (kX == kDecPrepared)
    dec_load_prepared(L, G, sq, s_sx, s_rs);
  else if (kX == kDecRms)
    dec_rms_quantise(L, G, sq, s_sx, s_rs, s_amax, s_ss, s_ms, s_flag,
                     reinterpret_cast<unsigned long long*>(sq + L.q_bytes - kRmsBins * 8));
  if (kRegQuant) {
    if (!early_x) dec_quant_load<kX>(L, G, f);
    dec_quant_rest<kX>(L, G, f, sq, s_sx, s_rs, s_amax);
  }
  consumers_sync();  // codes, scales and row sums visible to every warp

  const int g = lane >> 2, t = lane & 3;
  int acc[4][MT][4];
  float dg0 = 0.0f, dg1 = 0.0f;  // row scales of the current task
  auto zero_acc = [&]() {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[cc][mt][k] = 0;
  };
  zero_acc();
  int qp = -1, qlane[MT];  // the lane's token-row offset, for problem qp
  // Contract one group from its registers into acc; at the end of its task,
  // write the task's result. False if a wait gave up.
  auto run = [&](const DecRun& Gr, const uint8_t* stage) -> bool {
    const struct {
      int p, i, j;
    } T{Gr.p(), Gr.i, Gr.j()};
    const DecProblem& P = L.pr[T.p];
    if (!kAccOut && Gr.first()) {
      const float2 dd = *reinterpret_cast<const float2*>(stage + 16 * RS + 8 * lane);
      dg0 = dd.x;
      dg1 = dd.y;
    }
    // Lanes of token columns past M read the last token's codes (their MMA
    // columns are never used).
    if (T.p != qp) {
      qp = T.p;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int m = g + 8 * mt < P.M ? g + 8 * mt : P.M - 1;
        qlane[mt] = m * P.q_stride + 32 * t;
      }
    }
    const uint8_t* qb[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) qb[mt] = sq + Gr.qoff + qlane[mt];
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
      if (k < Gr.n()) {
        // rows g and g + 8 have the same parity, hence the same chunk order
        const int cpos = 16 * dec_chunk_pos<UPT>(g, 4 * k + t);
        const uint4 va = *reinterpret_cast<const uint4*>(stage + g * RS + cpos);
        const uint4 vb = *reinterpret_cast<const uint4*>(stage + (g + 8) * RS + cpos);
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 Q[MT][2];
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint8_t* qp = qb[mt] + 256 * k + 128 * h;
            Q[mt][0] = *reinterpret_cast<const uint4*>(qp);
            Q[mt][1] = *reinterpret_cast<const uint4*>(qp + 16);
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t mask = 0x03030303u << (2 * cc);
            const uint32_t a0 = wa[2 * h] & mask, a2 = wa[2 * h + 1] & mask;
            const uint32_t a1 = wb[2 * h] & mask, a3 = wb[2 * h + 1] & mask;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              // class cc of words 2h (b0) and 2h+1 (b1): an aligned register pair
              const uint32_t b0 = cc == 0 ? Q[mt][0].x : (cc == 1 ? Q[mt][0].z : (cc == 2 ? Q[mt][1].x : Q[mt][1].z));
              const uint32_t b1 = cc == 0 ? Q[mt][0].y : (cc == 1 ? Q[mt][0].w : (cc == 2 ? Q[mt][1].y : Q[mt][1].w));
              dec_mma(acc[cc][mt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
      }
    }
    if (!Gr.last()) return true;
    const int gt = t0 + T.i;
    const int row0 = (gt - P.tile0) * 16;
    const int rv = P.N - row0 < 16 ? P.N - row0 : 16;
    // Slot s serves tiles s, s + 16, s + 32, ... in turn; a tile may use it
    // once the tile 16 before it has finished (s_gen counts finished turns).
    const int s = T.i % kDecodeSlots;
    const int gen = T.i / kDecodeSlots;
    if (*reinterpret_cast<volatile int32_t*>(&s_gen[s]) != gen) {
      const uint64_t w0 = globaltimer_ns();
      while (*reinterpret_cast<volatile int32_t*>(&s_gen[s]) != gen) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - w0 > kWaitLimitNs) {
          *abort_flag = 1;
          if (L.err != nullptr) atomicCAS(L.err, 0u, (uint32_t)kDevTimeoutMma);
          return false;
        }
      }
      __threadfence_block();
    }
    if (P.nchunk == 1) {
      // The warp holds the whole tile: lane (g, t) has rows g and g+8 for
      // tokens 2t, 2t+1 (+ 8 per token group). Class c holds 4^c * sum
      // q*(code+1), an exact multiple of 4^c. y = RN(RN(a / s_x) * D), the
      // quotient by the IEEE fp32 division of the exact float(a).
      const int M = P.M;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (M == 1 && (k & 1)) continue;  // one token: only the even columns exist
          const int tok = 8 * mt + 2 * t + (k & 1);
          const int r = g + 8 * (k >> 1);
          if (tok < M && r < rv) {
            const int a = acc[0][mt][k] + (acc[1][mt][k] >> 2) + (acc[2][mt][k] >> 4) + (acc[3][mt][k] >> 6) -
                          s_rs[T.p * 16 + tok];
            const int64_t o = (int64_t)tok * P.N + row0 + r;
            if (kAccOut)
              P.acc[o] = a;
            else
              P.y[o] = rescale(a, s_sx[T.p * 16 + tok], (k >> 1) ? dg1 : dg0);
          }
        }
      zero_acc();
      // The slot was not used: pass its turn on (no shared data to order).
      __syncwarp();
      if (lane == 0) *reinterpret_cast<volatile int32_t*>(&s_gen[s]) = gen + 1;
      return true;
    }
    // Chunked tile: partial sums through the slot's block.
    if (!kAccOut && T.j == 0 && lane < 16) s_D[s * 16 + lane] = dg0;
    // Partial sums of this chunk into the tile's block.
    int32_t* blk = s_acc + s * 16 * AC;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int tok = 8 * mt + 2 * t + (k & 1);
        if (tok < P.M) {
          const int v = acc[0][mt][k] + (acc[1][mt][k] >> 2) + (acc[2][mt][k] >> 4) + (acc[3][mt][k] >> 6);
          atomicAdd(blk + (g + 8 * (k >> 1)) * AC + tok, v);
        }
      }
    zero_acc();
    __syncwarp();
    __threadfence_block();
    int last = 0;
    if (lane == 0) last = atomicAdd(&s_cnt[s], 1) == P.nchunk - 1;
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (last) {
      // Every chunk of the tile is in: outputs, then hand the slot on.
      __threadfence_block();
      for (int idx = lane; idx < 16 * P.M; idx += 32) {
        const int tok = idx >> 4, r = idx & 15;
        if (r < rv) {
          const int a = blk[r * AC + tok] - s_rs[T.p * 16 + tok];
          const int64_t o = (int64_t)tok * P.N + row0 + r;
          if (kAccOut)
            P.acc[o] = a;
          else
            P.y[o] = rescale(a, s_sx[T.p * 16 + tok], s_D[s * 16 + r]);
        }
      }
      __syncwarp();
      for (int k = lane; k < 16 * AC; k += 32) blk[k] = 0;
      if (lane == 0) s_cnt[s] = 0;
      __syncwarp();
      __threadfence_block();
      if (lane == 0) *reinterpret_cast<volatile int32_t*>(&s_gen[s]) = gen + 1;
    }
    return true;
  };
  // All S stages were filled before the quantiser ran. Wait for the oldest,
  // contract it, refill its stage with the next group: S - 1 groups stay in
  // flight during each contraction. (The stage's shared loads have all been
  // consumed by the MMAs of the contraction before the refill is issued.)
  int st = 0;
#pragma unroll 1
  for (;;) {
    cp_async_wait<S - 1>();
    __syncwarp();  // every lane's copies of this stage have landed
    const DecRun R = st ? rec1 : rec0;
    if (!R.valid() || !run(R, wstage + st * SB)) break;
    __syncwarp();
    const DecRun Rn = cur.issue(L, t0, nt, wstage + st * SB, lane);
    cp_async_commit();
    if (st) rec1 = Rn; else rec0 = Rn;
    st ^= 1;
  }
  cp_async_wait<0>();  // no copy is left in flight when the warp exits
}

using DecKernel = void (*)(const DecLaunch);

// The decode kernel for (MT, output kind, input mode), with its dynamic
// shared-memory limit raised (once per device).
template <int MT, bool kAccOut, int kX>
static cudaError_t decode_kernel(DecKernel* out) {
  static std::atomic<bool> raised[64];
  DecKernel kern = bl_ternary_decode_kernel<MT, kAccOut, kX>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !raised[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDecodeSmemMax);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev].store(true, std::memory_order_release);
  }
  *out = kern;
  return cudaSuccess;
}

int64_t decode_q_stride(int64_t K) { return ((K + 255) / 256) * 256 + 16; }

static int64_t round128(int64_t v) { return (v + 127) / 128 * 128; }

// Shared-memory bytes of a launch (q_total includes the RMSNorm mode's
// exact-sum bins, which follow the codes), or -1 when it does not fit.
static int64_t decode_smem(int64_t q_total, int64_t maxM) {
  const int64_t stages = (int64_t)kDecWarps * kDecStages * dec_stage_bytes<dec_upt<1>()>();
  const int64_t total = stages + q_total + dec_fixed_bytes((int)maxM, kDecStages);
  return total <= kDecodeSmemMax ? total : -1;
}

bool decode_group_fits(const DecCall* calls, int n) {
  if (n < 1 || n > kDecodeMaxGroup) return false;
  int64_t q = 0, maxM = 0;
  for (int i = 0; i < n; ++i) {
    if (calls[i].M < 1 || calls[i].M > kDecodeMaxM) return false;
    q += round128(calls[i].M * decode_q_stride(calls[i].K));
    maxM = calls[i].M > maxM ? calls[i].M : maxM;
  }
  return decode_smem(q, maxM) >= 0;
}

bool decode_fits(int64_t M, int64_t K, bool rms) {
  if (M < 1 || M > kDecodeMaxM) return false;
  const int64_t q = round128(M * decode_q_stride(K)) + (rms ? kRmsBins * 8 : 0);
  return decode_smem(q, M) >= 0;
}

// Split the launch's tiles into `grid` contiguous ranges of about equal bytes,
// at least one tile each. A problem's tiles all hold 16 rows of the same
// length (its last tile possibly fewer rows), so the boundary nearest to each
// 1/grid of the bytes is computed directly, problem by problem: O(grid +
// problems) host work per launch.
static void partition_by_bytes(DecLaunch& LP, int grid) {
  const DecHead& L = LP.h;
  int* cta_start = LP.cta_start;
  int64_t total = 0;
  int64_t pre[kDecodeMaxGroup + 1];
  pre[0] = 0;
  for (int p = 0; p < L.nprob; ++p) {
    pre[p + 1] = pre[p] + (int64_t)L.pr[p].N * L.pr[p].wpr * 4;
    total = pre[p + 1];
  }
  cta_start[0] = 0;
  int p = 0;
  for (int c = 1; c < grid; ++c) {
    const int64_t target = total * c / grid;
    while (p + 1 < L.nprob && pre[p + 1] <= target) ++p;
    const DecProblem& P = L.pr[p];
    const int64_t tb = 64 * (int64_t)P.wpr;  // bytes of a full tile
    int64_t k = tb > 0 ? (target - pre[p] + tb / 2) / tb : 0;
    if (k > P.tiles) k = P.tiles;
    int gt = P.tile0 + (int)k;
    // Strictly increasing, and enough tiles left for the CTAs after this one.
    if (gt <= cta_start[c - 1]) gt = cta_start[c - 1] + 1;
    if (gt > L.total_tiles - (grid - c)) gt = L.total_tiles - (grid - c);
    cta_start[c] = gt;
  }
  cta_start[grid] = L.total_tiles;
}

cudaError_t launch_decode(const DecCall* calls, int n, int input, const float* g, float eps, uint32_t* err, bool pdl,
                          cudaStream_t stream, int num_sms) {
  if (n < 1 || n > kDecodeMaxGroup) return cudaErrorInvalidValue;
  if ((input == kDecRms || input == kDecPrepared) && n != 1) return cudaErrorInvalidValue;
  DecLaunch LP;
  std::memset(&LP, 0, sizeof(LP));
  DecHead& L = LP.h;
  int64_t maxM = 0, q = 0;
  int tiles = 0;
  for (int i = 0; i < n; ++i) {
    if (calls[i].M < 1 || calls[i].M > kDecodeMaxM || calls[i].N < 1) return cudaErrorInvalidValue;
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
  }
  const int MT = maxM <= 8 ? 1 : 2;
  if (input == kDecRms) q += kRmsBins * 8;  // exact-sum bins after the codes
  int64_t smem = decode_smem(q, maxM);
  if (smem < 0) return cudaErrorInvalidValue;
  L.acc_cols = (int)maxM;
  L.nprob = n;
  L.total_tiles = tiles;
  L.q_bytes = (int)q;
  L.err = err;
  L.g = g;
  L.eps = eps;
  const bool accout = calls[0].acc != nullptr;
  for (int i = 1; i < n; ++i)
    if ((calls[i].acc != nullptr) != accout) return cudaErrorInvalidValue;  // one output kind per launch
  DecKernel kern = nullptr;
  cudaError_t e = cudaErrorInvalidValue;
#define BL_DEC(MTV, AO, XM) \
  if (MT == MTV && accout == AO && input == XM) e = decode_kernel<MTV, AO, XM>(&kern);
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
  if (e != cudaSuccess) return e;
  // One CTA per SM leaves room on every SM for a CTA of the next launch
  // (programmatic dependent launch), which matters for short launches. Long
  // streams take as many CTAs per SM as fit (more copies in flight).
  int per_sm = 1;
  if (tiles >= 8 * num_sms) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, (size_t)smem);
    if (e != cudaSuccess) return e;
    per_sm = per_sm < 1 ? 1 : (per_sm > 3 ? 3 : per_sm);
  }
  int grid = per_sm * num_sms;
  if (grid > tiles) grid = tiles;
  if (grid > kDecMaxGrid) grid = kDecMaxGrid;
  partition_by_bytes(LP, grid);
  // Tasks: whole tiles when every warp of a CTA gets two or more of them (a
  // warp then writes its tiles' outputs itself); otherwise chunks. A launch
  // of one problem cuts its tiles into chunks of one group of units, which
  // spreads a CTA's share evenly over its warps; a launch of several problems
  // uses chunks of about nu * tiles_per_cta / 8 units (on the B200, measured
  // faster there: fewer chunks to combine through shared memory).
  const double tiles_per_cta = (double)tiles / grid;
  for (int i = 0; i < n; ++i) {
    DecProblem& P = L.pr[i];
    int upt = P.nu;
    if (tiles_per_cta < 2.0 * kDecWarps) {
      upt = n == 1 ? dec_upt<1>() : (int)((P.nu * tiles_per_cta + kDecWarps - 1) / kDecWarps);
      upt = upt < 1 ? 1 : (upt > P.nu ? P.nu : upt);
    }
    P.upt = upt;
    P.nchunk = (P.nu + upt - 1) / upt;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  L.pdl = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, LP);
}

}  // namespace bl
