// bl_gemm.cu - prefill GEMM (M > 16 tokens) on the 5th-generation tensor cores.
//
// Computes acc[m,n] = sum_k q[m,k] * code[n,k] and the rescale of
// "Core AI model zoo - BitVLA", sections 1-2 (y = F.linear(ActQuant(x),
// WeightQuant(W)) with the per-row scale D [N,1]). The pages only give an
// M=1 decode kernel; a prefill of many tokens is a dense int8 contraction, so
// it runs on tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Tile: 128 weight rows (MMA M) x 192 tokens (MMA N); 256 codes per pipeline
// stage (8 MMAs of K=32 per barrier round trip, so the single issuing thread
// keeps the tensor pipe fed). Larger MMAs carry the pipe's per-instruction
// cost over more work: measured on gate_up (M=4096), a 128x192x32 MMA issues
// every ~155-185 cycles against ~144 for 128x128x32.
//
// Operand placement (chosen for shared-memory bandwidth):
//   A = unpacked ternary weights, written by four unpack warps straight from
//       registers into TMEM (tcgen05.st). `(w >> 2c) & 0x03030303` yields
//       code+1 for columns {c, 4+c, 8+c, 12+c} of a packed word, so TMEM
//       holds each 16-column group in the order 4c+b <- 4b+c. Two stages.
//   B = int8 activations in the same order (written so by the ActQuant
//       kernel), loaded by TMA as 192 tokens x 128 bytes with 128-byte
//       swizzle; three stages, a ring of its own.
//   D = int32 accumulators in TMEM, two buffers of 192 columns
//       (2*192 + 2*64 = 512 columns with the A stages).
// Warp roles: 0 TMA producer, 1 MMA issuer (TMEM owner), 2 per-token
// constants (s_x and sum_k q) into a shared ring, 4..7 unpack, 8..15
// epilogue. An epilogue warp owns 32 rows x 96 tokens of the accumulator and
// walks it in chunks of 32 tokens: TMEM load, rescale y = RN(RN(acc/s_x)*D),
// a 4 KB staging buffer (two per warp, alternating) and one TMA bulk store
// per chunk (plain stores when N % 4 != 0); the TMEM buffer is released once
// its last chunk is in registers.
// Every barrier wait is bounded in time; a timeout sets a shared abort flag
// and the error word in the workspace, and all roles drain and exit.
#include "bl_internal.h"

#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

namespace bl {

constexpr int kBM = 128;   // weight rows per tile (MMA M)
constexpr int kBK = 256;   // codes per stage
constexpr int kStageWords = kBK / 16;          // packed words per row per stage
constexpr int kACols = kBK / 4;                // TMEM columns of one A stage
constexpr int kBBoxes = kBK / 128;             // TMA boxes per B stage
constexpr uint32_t kTmemCols = 512;
constexpr int kAccCol = 0;                     // accumulator b at column BN*b

// Tile shapes: BN tokens per tile (MMA N). 192 tokens carry the pipe's
// per-instruction cost over more work; 128 tokens waste less on launches of
// one or two tiles per CTA, whose pipeline fill and last epilogue are not
// overlapped. TMEM holds the two accumulators and the A stages.
template <int BN>
struct GemmShape {
  static constexpr int kBN = BN;
  static constexpr int kAStages = BN == 128 ? 4 : 2;  // ring of A stages in TMEM
  static constexpr int kBStages = BN == 128 ? 4 : 3;  // ring of B stages in shared memory
  static constexpr uint32_t kBBoxBytes = BN * 128;    // one TMA box: BN tokens x 128 codes
  static constexpr uint32_t kBStageBytes = kBBoxes * kBBoxBytes;
  static constexpr int kACol = 2 * BN;                // A stage s at column 2*BN + kACols*s
  static constexpr int kEpiTokens = BN / 2;           // tokens per epilogue warp
  static_assert(kACol + kAStages * kACols <= (int)kTmemCols, "TMEM budget");
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N for M = 128");
  static_assert(kBBoxBytes % 1024 == 0, "128-byte swizzle atoms");
};

constexpr int kWarpConst = 2;
constexpr int kUnpackWarp0 = 4;                // 4..7: one per TMEM lane quarter
constexpr int kEpiWarp0 = 8;                   // 8..15: two per lane quarter
constexpr int kEpiWarps = 8;
constexpr int kEpiChunk = 32;                  // accumulator columns per TMEM load
constexpr int kGemmThreads = 32 * (kEpiWarp0 + kEpiWarps);  // 512
constexpr int kUnpackPrefetch = 2;             // stages of packed words in flight
constexpr int kConstRing = 4;                  // tiles of per-token constants in flight
constexpr uint32_t kYChunkBytes = kEpiChunk * 32 * 4;  // one epilogue chunk: 32 tokens x 32 rows fp32

struct TokConst {
  float sx;    // s_x = 127 / max|x|
  float rx;    // RN(1 / s_x), for the rescale's corrected division
  int32_t rs;  // sum_k q[m, k]
};

template <int BN>
struct GemmSmem {
  static constexpr int kAStages = GemmShape<BN>::kAStages;
  static constexpr int kBStages = GemmShape<BN>::kBStages;
  uint64_t full_b[kBStages];   // activation stage landed (TMA bytes)
  uint64_t empty_b[kBStages];  // activation stage consumed (MMA commit)
  uint64_t full_a[kAStages];   // weight stage written to TMEM (4 unpack warps)
  uint64_t empty_a[kAStages];  // weight stage consumed (MMA commit)
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t cst_full[kConstRing];
  uint64_t cst_empty[kConstRing];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  TokConst cst[kConstRing][BN];
};

struct GemmParams {
  const uint32_t* packed;
  const float* D;
  const float* s_x;
  const int32_t* rowsum;
  float* y;
  int32_t* acc_out;
  uint32_t* err;
  int M;
  int N;
  int K;
  int wpr;         // packed words in the contracted K range of a row
  int wstride;     // words from one row of `packed` to the next (>= wpr)
  int dstride;     // floats from D[n] to D[n + 1]
  int accumulate;  // add the rescaled tile to y (y = RN(y + t)) instead of storing it
  int kblocks;
  int tiles_n;
  int num_tiles;
};

// Smem: [B stages | Y chunks (two per epilogue warp) | GemmSmem], 1024-aligned;
// one CTA per SM (each CTA owns all 512 TMEM columns).
constexpr size_t kSmemY = (size_t)kEpiWarps * 2 * kYChunkBytes;
template <int BN>
constexpr size_t gemm_smem_b() { return (size_t)GemmShape<BN>::kBStages * GemmShape<BN>::kBStageBytes; }
template <int BN>
constexpr size_t gemm_smem_bytes() {
  return 1024 + gemm_smem_b<BN>() + kSmemY + ((sizeof(GemmSmem<BN>) + 127) & ~size_t(127));
}
static_assert(gemm_smem_bytes<128>() <= 227 * 1024 && gemm_smem_bytes<192>() <= 227 * 1024, "shared memory");

// Warp-uniform bounded wait: lane 0 polls, the whole warp gets the outcome, so
// the warp stays converged for the .sync.aligned tcgen05 instructions.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                          uint32_t code) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, err, code) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  return ok != 0;
}

// Position in this CTA's job sequence (tile-major, k-block-minor), advanced
// without integer divisions.
struct JobCursor {
  int tile_local;
  int kb;
  __device__ __forceinline__ void next(int kblocks) {
    if (++kb == kblocks) {
      kb = 0;
      ++tile_local;
    }
  }
};

template <bool kAligned>
__device__ __forceinline__ void unpack_load(const GemmParams& p, const JobCursor& jc, int row_in_tile,
                                            uint32_t (&w)[kStageWords]) {
  const int tile = blockIdx.x + jc.tile_local * gridDim.x;
  const int64_t n = (int64_t)(tile % p.tiles_n) * kBM + row_in_tile;
  const int w0 = jc.kb * kStageWords;
  if (n < p.N) {
    const uint32_t* rp = p.packed + n * (int64_t)p.wstride + w0;
    if (kAligned) {
      // wpr % 4 == 0 and w0 % 4 == 0: each group of four words is all in or all out.
#pragma unroll
      for (int q = 0; q < kStageWords / 4; ++q) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (w0 + 4 * q < p.wpr) v = __ldg(reinterpret_cast<const uint4*>(rp) + q);
        w[4 * q] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kStageWords; ++j) w[j] = (w0 + j < p.wpr) ? __ldg(rp + j) : 0u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kStageWords; ++j) w[j] = 0u;
  }
}

template <int BN, bool kAligned, bool kAccOut, bool kTmaStore>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_out,
                const GemmParams p) {
  using Shape = GemmShape<BN>;
  constexpr int kBN = Shape::kBN;
  constexpr int kAStages = Shape::kAStages;
  constexpr int kBStages = Shape::kBStages;
  constexpr uint32_t kBBoxBytes = Shape::kBBoxBytes;
  constexpr uint32_t kBStageBytes = Shape::kBStageBytes;
  constexpr int kACol = Shape::kACol;
  constexpr int kEpiTokens = Shape::kEpiTokens;
  static_assert(kEpiTokens % kEpiChunk == 0, "epilogue chunks");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  uint8_t* sY = smem + gemm_smem_b<BN>();
  GemmSmem<BN>& S = *reinterpret_cast<GemmSmem<BN>*>(smem + gemm_smem_b<BN>() + kSmemY);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int my_tiles = p.num_tiles > (int)blockIdx.x ? (p.num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int jobs = my_tiles * p.kblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&S.full_b[s], 1);   // the TMA producer's expect-tx arrival
      mbar_init(&S.empty_b[s], 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&S.full_a[s], 4);   // one unpack warp per TMEM lane quarter
      mbar_init(&S.empty_a[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_empty[b], kEpiWarps);
    }
    for (int r = 0; r < kConstRing; ++r) {
      mbar_init(&S.cst_full[r], 1);
      mbar_init(&S.cst_empty[r], kEpiWarps);
    }
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_q);
    if (kTmaStore) tma_prefetch_desc(&tmap_out);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  volatile int* abort_flag = &S.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (x)
    if (lane == 0) {
      // The quantised activations come from the launch this one may overlap
      // (programmatic dependent launch): wait for it before the first load.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int s = 0;
      uint32_t ph = 0;
      JobCursor c{0, 0};
      int issued = 0;
      for (int j = 0; j < jobs; ++j) {
        if (!mbar_wait(&S.empty_b[s], ph ^ 1, abort_flag, p.err, kDevTimeoutProducer)) break;
        const int tile = blockIdx.x + c.tile_local * gridDim.x;
        const int m0 = (tile / p.tiles_n) * kBN;
        const int k0 = c.kb * kBK;
        // A box lying wholly past K is not loaded: its A codes are zero, so
        // whatever the stage buffer holds there contributes nothing.
        int nbox = (p.K - k0 + 127) / 128;
        nbox = nbox > kBBoxes ? kBBoxes : nbox;
        mbar_arrive_expect_tx(&S.full_b[s], (uint32_t)nbox * kBBoxBytes);
        for (int b = 0; b < nbox; ++b)
          tma_load_2d(sB + (size_t)s * kBStageBytes + b * kBBoxBytes, &tmap_q, k0 + 128 * b, m0, &S.full_b[s]);
        ++issued;
        c.next(p.kblocks);
        if (++s == kBStages) {
          s = 0;
          ph ^= 1;
        }
      }
      // Let every issued copy land before the CTA can exit.
      const int first = issued > kBStages ? issued - kBStages : 0;
      for (int j = first; j < issued; ++j)
        mbar_wait(&S.full_b[j % kBStages], (j / kBStages) & 1, nullptr, p.err, kDevTimeoutDrain, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kBM, kBN);
      const uint64_t bdesc0 = umma_sdesc_sw128(sB);
      int sb = 0, sa = 0;
      uint32_t phb = 0, pha = 0;
      bool ok = true;
      for (int lt = 0; lt < my_tiles && ok; ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&S.acc_empty[b], ((lt >> 1) & 1) ^ 1, abort_flag, p.err, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kAccCol + kBN * b;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&S.full_a[sa], pha, abort_flag, p.err, kDevTimeoutMma) ||
              !mbar_wait(&S.full_b[sb], phb, abort_flag, p.err, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem + kACol + kACols * sa;
          // K=32 steps of this stage that hold real codes (the rest are zero).
          const int rem = p.K - kb * kBK;
          const int steps = rem >= kBK ? kBK / 32 : (rem + 31) / 32;
#pragma unroll
          for (int k8 = 0; k8 < kBK / 32; ++k8) {
            if (k8 < steps) {
              const uint64_t bdesc = bdesc0 + (uint64_t)((sb * kBStageBytes + (k8 >> 2) * kBBoxBytes) >> 4) +
                                     2 * (k8 & 3);
              umma_i8_ts(d_tmem, a_tmem + 8 * k8, bdesc, idesc, (kb | k8) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&S.empty_a[sa]);
          tc_commit(&S.empty_b[sb]);
          if (++sa == kAStages) {
            sa = 0;
            pha ^= 1;
          }
          if (++sb == kBStages) {
            sb = 0;
            phb ^= 1;
          }
        }
        if (ok) tc_commit(&S.acc_full[b]);
      }
      // All issued MMAs complete before TMEM is released.
      tc_commit(&S.drain);
      mbar_wait(&S.drain, 0, nullptr, p.err, kDevTimeoutDrain, 100000000ull);
    }
  } else if (warp == kWarpConst) {
    // ------------------------------------------------ per-token constants, ahead of the epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");  // s_x and row sums come from the same launch
    int r = 0;
    uint32_t ph = 0;
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int tile = blockIdx.x + lt * gridDim.x;
      const int m0 = (tile / p.tiles_n) * kBN;
      float sx[kBN / 32];
      int32_t rs[kBN / 32];
#pragma unroll
      for (int h = 0; h < kBN / 32; ++h) {
        const int m = m0 + 32 * h + lane;
        const bool ok = m < p.M;
        sx[h] = ok ? p.s_x[m] : 1.0f;  // plain loads: written by the grid waited for
        rs[h] = ok ? p.rowsum[m] : 0;
      }
      if (!warp_wait(&S.cst_empty[r], ph ^ 1, abort_flag, p.err, kDevTimeoutEpilogue)) break;
#pragma unroll
      for (int h = 0; h < kBN / 32; ++h) {
        S.cst[r][32 * h + lane].sx = sx[h];
        S.cst[r][32 * h + lane].rx = __fdiv_rn(1.0f, sx[h]);
        S.cst[r][32 * h + lane].rs = rs[h];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.cst_full[r]);
      if (++r == kConstRing) {
        r = 0;
        ph ^= 1;
      }
    }
  } else if (warp >= kUnpackWarp0 && warp < kUnpackWarp0 + 4) {
    // ------------------------------------------------ A unpackers: one weight row per thread
    const int quarter = warp & 3;  // TMEM lane quarter (hardware rule: warp id % 4)
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    JobCursor lc{0, 0};
    uint32_t buf[kUnpackPrefetch][kStageWords];
#pragma unroll
    for (int q = 0; q < kUnpackPrefetch; ++q) {
      if (q < jobs) unpack_load<kAligned>(p, lc, row_in_tile, buf[q]);
      lc.next(p.kblocks);
    }
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int j0 = 0; j0 < jobs && ok; j0 += kUnpackPrefetch) {
#pragma unroll
      for (int q = 0; q < kUnpackPrefetch; ++q) {
        const int j = j0 + q;
        if (j >= jobs) break;
        if (!warp_wait(&S.empty_a[s], ph ^ 1, abort_flag, p.err, kDevTimeoutUnpack)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < kStageWords / 8; ++h) {
          uint32_t v[32];
#pragma unroll
          for (int w = 0; w < 8; ++w)
#pragma unroll
            for (int c = 0; c < 4; ++c) v[4 * w + c] = (buf[q][8 * h + w] >> (2 * c)) & 0x03030303u;
          tmem_st_32x32b_x32(lane_base + kACol + kACols * s + 32 * h, v);
        }
        if (j + kUnpackPrefetch < jobs) unpack_load<kAligned>(p, lc, row_in_tile, buf[q]);
        lc.next(p.kblocks);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.full_a[s]);
        if (++s == kAStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue: 32 weight rows x kEpiTokens tokens per warp
    const int ew = warp - kEpiWarp0;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t* sy0 = reinterpret_cast<uint32_t*>(sY + (size_t)ew * 2 * kYChunkBytes);
    int ybuf = 0;  // which of the warp's two staging chunks the next chunk uses
    int r = 0;
    uint32_t rph = 0;
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int b = lt & 1;
      const int tile = blockIdx.x + lt * gridDim.x;
      const int m0 = (tile / p.tiles_n) * kBN + kEpiTokens * half;
      const int n0 = (tile % p.tiles_n) * kBM + quarter * 32;
      const int64_t n = (int64_t)n0 + lane;
      const bool nvalid = n < p.N;
      const float dn = (!kAccOut && nvalid) ? __ldg(p.D + n * p.dstride) : 0.0f;
      if (!warp_wait(&S.acc_full[b], (lt >> 1) & 1, abort_flag, p.err, kDevTimeoutEpilogue)) break;
      tc_fence_after();
      if (!warp_wait(&S.cst_full[r], rph, abort_flag, p.err, kDevTimeoutEpilogue)) break;
      const TokConst* cst = &S.cst[r][kEpiTokens * half];
      // Chunks of 32 accumulator columns: load, rescale, store. Lane `lane`
      // holds row n of the chunk's 32 tokens. With TMA stores the chunk is
      // staged in one of the warp's two shared buffers and written as one
      // 32 x 32 box (rows past M or N are clipped); otherwise a warp's store
      // of one token covers 32 consecutive outputs (128 bytes).
#pragma unroll 1
      for (int c0 = 0; c0 < kEpiTokens; c0 += kEpiChunk) {
        uint32_t v[kEpiChunk];
        tmem_ld_32x32b_x32(lane_base + kAccCol + kBN * b + kEpiTokens * half + c0, v);
        tmem_wait_ld();
        if (c0 + kEpiChunk == kEpiTokens) {
          // The whole accumulator is in registers: hand the TMEM buffer back.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.acc_empty[b]);
        }
        uint32_t* sy = sy0 + ybuf * (kYChunkBytes / 4);
        if (kTmaStore) {
          // The store that used this buffer two chunks ago must have read it.
          if (lane == 0) bulk_wait_group_read1();
          __syncwarp();
        }
#pragma unroll
        for (int t = 0; t < kEpiChunk; ++t) {
          const TokConst kc = cst[c0 + t];
          const int a = (int)v[t] - kc.rs;
          const uint32_t out = kAccOut ? (uint32_t)a : __float_as_uint(rescale_rcp(a, kc.sx, kc.rx, dn));
          if (kTmaStore) {
            sy[t * 32 + lane] = out;
          } else {
            const int m = m0 + c0 + t;
            if (m < p.M && nvalid) {
              if (kAccOut) {
                p.acc_out[(int64_t)m * p.N + n] = (int32_t)out;
              } else if (p.accumulate) {
                float* py = p.y + (int64_t)m * p.N + n;  // one writer per element in this launch
                *py = __fadd_rn(*py, __uint_as_float(out));
              } else {
                __stcs(p.y + (int64_t)m * p.N + n, __uint_as_float(out));
              }
            }
          }
        }
        if (kTmaStore) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (!kAccOut && p.accumulate)
              tma_reduce_add_2d(&tmap_out, n0, m0 + c0, sy);
            else
              tma_store_2d(&tmap_out, n0, m0 + c0, sy);
            bulk_commit_group();
          }
          ybuf ^= 1;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.cst_empty[r]);
      if (++r == kConstRing) {
        r = 0;
        rph ^= 1;
      }
    }
    if (kTmaStore) {
      if (lane == 0) bulk_wait_group0();
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host --
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

template <int BN, bool kAligned, bool kAccOut, bool kTmaStore>
static cudaError_t launch_gemm_t(const CUtensorMap& tq, const CUtensorMap& to, const GemmParams& p, int grid,
                                 cudaStream_t stream) {
  auto kern = gemm_kernel<BN, kAligned, kAccOut, kTmaStore>;
  constexpr size_t smem = gemm_smem_bytes<BN>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch: TMEM allocation, barrier setup and the
  // weight unpack (which needs nothing from the previous launch) overlap the
  // quantiser that precedes this launch; the activation loads and the
  // per-token constants wait for it (griddepcontrol.wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, to, p);
}

// Estimated time of a launch with BN-token tiles, in units of 10 ns on the
// B200 (fitted to timings of the prefill and SigLIP shapes): the waves of
// tiles times a tile's k-blocks at the measured cost of one k-block, plus
// the launch's fixed cost (pipeline fill and the last tile's epilogue, which
// nothing overlaps; larger for 192-token tiles).
static int64_t gemm_estimate(int BN, int64_t M, int64_t tiles_n, int64_t kblocks, int grid) {
  const int64_t tiles = (M + BN - 1) / BN * tiles_n;
  const int64_t waves = (tiles + grid - 1) / grid;
  return BN == 128 ? waves * kblocks * 80 + 750 : waves * kblocks * 95 + 1390;
}

cudaError_t launch_gemm(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                        int32_t* acc_out, void* ws, cudaStream_t stream, int num_sms) {
  GemmSlice sl;
  sl.k0 = 0;
  sl.kfull = K;
  sl.dstride = 1;
  sl.accumulate = false;
  sl.rowsum = nullptr;
  return launch_gemm_slice(M, N, K, sl, packed, D, y, acc_out, ws, stream, num_sms);
}

cudaError_t launch_gemm_slice(int64_t M, int64_t N, int64_t K, const GemmSlice& sl, const uint32_t* packed,
                              const float* D, float* y, int32_t* acc_out, void* ws, cudaStream_t stream,
                              int num_sms) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  int8_t* q = reinterpret_cast<int8_t*>(base + ws_q_off(M)) + sl.k0;
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  // Token-tile width: whichever the cost model puts first.
  const int64_t tiles_n = (N + kBM - 1) / kBM;
  const int64_t kblocks = (K + kBK - 1) / kBK;
  const int est_grid = num_sms;
  const int BN = gemm_estimate(192, M, tiles_n, kblocks, est_grid) < gemm_estimate(128, M, tiles_n, kblocks, est_grid)
                     ? 192
                     : 128;
  CUtensorMap tmap_q, tmap_out;
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)sl.kfull};
    const cuuint32_t box[2] = {128u, (cuuint32_t)BN};
    const cuuint32_t estride[2] = {1, 1};
    if (encode(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // Output via TMA bulk stores when every output row starts on a 16-byte boundary.
  void* out = acc_out != nullptr ? static_cast<void*>(acc_out) : static_cast<void*>(y);
  const bool tma_store = (N % 4) == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  std::memset(&tmap_out, 0, sizeof(tmap_out));
  if (tma_store) {
    const cuuint64_t gdim[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)N * 4};
    const cuuint32_t box[2] = {32u, (cuuint32_t)kEpiChunk};
    const cuuint32_t estride[2] = {1, 1};
    if (encode(&tmap_out, acc_out != nullptr ? CU_TENSOR_MAP_DATA_TYPE_INT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               out, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }

  GemmParams p;
  p.packed = packed + sl.k0 / 16;
  p.D = D;
  p.s_x = reinterpret_cast<const float*>(base + ws_sx_off(M));
  p.rowsum = sl.rowsum != nullptr ? sl.rowsum : reinterpret_cast<const int32_t*>(base + ws_rowsum_off(M));
  p.y = y;
  p.acc_out = acc_out;
  p.err = reinterpret_cast<uint32_t*>(base);
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.wpr = (int)(K / 16);
  p.wstride = (int)(sl.kfull / 16);
  p.dstride = sl.dstride;
  p.accumulate = sl.accumulate ? 1 : 0;
  p.kblocks = (int)kblocks;
  p.tiles_n = (int)tiles_n;
  const int64_t tiles_m = (M + BN - 1) / BN;
  const int64_t nt = tiles_m * p.tiles_n;
  if (nt > 0x7FFFFFFF) return cudaErrorInvalidValue;
  p.num_tiles = (int)nt;
  const int grid = (int)(nt < num_sms ? nt : num_sms);
  const bool aligned = (p.wpr % 4) == 0 && (p.wstride % 4) == 0 && (reinterpret_cast<uintptr_t>(p.packed) & 15u) == 0;
  const bool accout = acc_out != nullptr;
#define BL_GEMM_CASE(AL, AO, TS)                                                                     \
  if (aligned == AL && accout == AO && tma_store == TS)                                              \
    return BN == 192 ? launch_gemm_t<192, AL, AO, TS>(tmap_q, tmap_out, p, grid, stream)               \
                     : launch_gemm_t<128, AL, AO, TS>(tmap_q, tmap_out, p, grid, stream);
  BL_GEMM_CASE(true, false, true)
  BL_GEMM_CASE(true, false, false)
  BL_GEMM_CASE(false, false, true)
  BL_GEMM_CASE(false, false, false)
  BL_GEMM_CASE(true, true, true)
  BL_GEMM_CASE(true, true, false)
  BL_GEMM_CASE(false, true, true)
  BL_GEMM_CASE(false, true, false)
#undef BL_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace bl
