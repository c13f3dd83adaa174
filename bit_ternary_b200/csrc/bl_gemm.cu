// bl_gemm.cu - prefill GEMM (M > 16 tokens) on the 5th-generation tensor cores.
//
// Computes acc[m,n] = sum_k q[m,k] * code[n,k] and the rescale of
// "Core AI model zoo - BitVLA", sections 1-2 (y = F.linear(ActQuant(x),
// WeightQuant(W)) with the per-row scale D [N,1]). The pages only give an
// M=1 decode kernel; a prefill of many tokens is a dense int8 contraction, so
// it runs on tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// Operand placement (chosen for shared-memory bandwidth):
//   A = unpacked ternary weights, 128 rows x 128 codes per stage, written by
//       four "unpack" warps straight from registers into TMEM (tcgen05.st).
//       The packed words are read from global memory; `(w >> 2c) & 0x03030303`
//       yields code+1 for columns {c, 4+c, 8+c, 12+c} of a word, so TMEM holds
//       the columns of every 16-column group in the order 4c+b <- 4b+c.
//   B = int8 activations in the same order (written so by the ActQuant
//       kernel), loaded by TMA as 128 tokens x 128 bytes with 128-byte swizzle.
//   D = int32 accumulators in TMEM, two buffers of 128 columns so the epilogue
//       of one tile overlaps the MMAs of the next.
// The MMA thread issues tcgen05.mma (M=128 weight rows, N=128 tokens, K=32)
// and signals stage reuse with tcgen05.commit. The epilogue warps read the
// accumulators with tcgen05.ld, subtract sum_k q (the +1 of the stored codes)
// and write y = RN(RN(acc/s_x)*D) with coalesced stores.
// Every barrier wait is bounded in time; a timeout sets a shared abort flag
// and the error word in the workspace, and all roles drain and exit.
#include "bl_internal.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace bl {

constexpr int kBM = 128;  // weight rows per tile (MMA M)
constexpr int kBN = 128;  // tokens per tile (MMA N)
constexpr int kBK = 128;  // codes per stage (4 MMAs of K=32)
constexpr int kAStages = 8;
constexpr int kBStages = 6;
constexpr int kGemmThreads = 512;  // 16 warps
constexpr int kEpiWarps = 8;       // warps 8..15: two per TMEM lane quarter, 64 tokens each
constexpr uint32_t kTmemCols = 512;
constexpr int kAccCol = 0;    // accumulator buffer b at column 128*b
constexpr int kACol = 256;    // A stage s at column 256 + 32*s
constexpr int kUnpackPrefetch = 4;
constexpr uint32_t kBStageBytes = kBN * kBK;  // 16 KB

struct GemmSmem {
  uint64_t b_full[kBStages];
  uint64_t b_empty[kBStages];
  uint64_t a_full[kAStages];
  uint64_t a_empty[kAStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  // Per-token epilogue constants, one private slice per epilogue warp:
  // 1/s_x in fp64 and sum_k q for the warp's 64 tokens.
  double tok_inv[kEpiWarps][64];
  int32_t tok_rs[kEpiWarps][64];
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
  int wpr;
  int kblocks;
  int tiles_n;
  int num_tiles;
};

// Smem: [B stages, 1024-aligned][GemmSmem]; padded so only one CTA fits per SM
// (each CTA allocates all 512 TMEM columns).
constexpr size_t kGemmSmemBytes = 1024 /*align slack*/ + (size_t)kBStages * kBStageBytes + sizeof(GemmSmem);
constexpr size_t kGemmSmemLaunch = kGemmSmemBytes > 120 * 1024 ? kGemmSmemBytes : 120 * 1024;

// Warp-uniform bounded wait: lane 0 polls, the whole warp gets its verdict, so
// the warp stays converged for the .sync.aligned tcgen05 instructions.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t* err,
                                          uint32_t code) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, err, code) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  return ok != 0;
}

template <bool kAligned>
__device__ __forceinline__ void unpack_load(const GemmParams& p, int job, int row_in_tile, uint32_t (&w)[8]) {
  const int tile_local = job / p.kblocks;
  const int kb = job - tile_local * p.kblocks;
  const int tile = blockIdx.x + tile_local * gridDim.x;
  const int tn = tile % p.tiles_n;
  const int64_t n = (int64_t)tn * kBM + row_in_tile;
  const int w0 = kb * (kBK / 16);
  if (n < p.N) {
    const uint32_t* rp = p.packed + n * (int64_t)p.wpr + w0;
    if (kAligned && w0 + 8 <= p.wpr) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(rp));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(rp + 4));
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = (w0 + j < p.wpr) ? __ldg(rp + j) : 0u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = 0u;
  }
}

template <bool kAligned, bool kAccOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_q, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(smem + (size_t)kBStages * kBStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int my_tiles = p.num_tiles > (int)blockIdx.x ? (p.num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&S.b_full[s], 1);
      mbar_init(&S.b_empty[s], 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&S.a_full[s], 4);
      mbar_init(&S.a_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_empty[b], kEpiWarps);
    }
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_q);
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
      int it = 0;
      bool ok = true;
      for (int lt = 0; lt < my_tiles && ok; ++lt) {
        const int tile = blockIdx.x + lt * gridDim.x;
        const int m0 = (tile / p.tiles_n) * kBN;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int s = it % kBStages;
          const uint32_t ph = (it / kBStages) & 1;
          if (!mbar_wait(&S.b_empty[s], ph ^ 1, abort_flag, p.err, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S.b_full[s], kBStageBytes);
          tma_load_2d(sB + (size_t)s * kBStageBytes, &tmap_q, kb * kBK, m0, &S.b_full[s]);
        }
      }
      // Let every issued copy land before the CTA can exit.
      const int first = it > kBStages ? it - kBStages : 0;
      for (int j = first; j < it; ++j)
        mbar_wait(&S.b_full[j % kBStages], (j / kBStages) & 1, nullptr, p.err, kDevTimeoutDrain, 100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kBM, kBN);
      int it = 0;
      bool ok = true;
      for (int lt = 0; lt < my_tiles && ok; ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&S.acc_empty[b], ((lt >> 1) & 1) ^ 1, abort_flag, p.err, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + kAccCol + 128 * b;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int sa = it % kAStages, sb = it % kBStages;
          if (!mbar_wait(&S.a_full[sa], (it / kAStages) & 1, abort_flag, p.err, kDevTimeoutMma) ||
              !mbar_wait(&S.b_full[sb], (it / kBStages) & 1, abort_flag, p.err, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = umma_sdesc_sw128(sB + (size_t)sb * kBStageBytes);
          const uint32_t a_tmem = tmem + kACol + 32 * sa;
#pragma unroll
          for (int k4 = 0; k4 < kBK / 32; ++k4)
            umma_i8_ts(d_tmem, a_tmem + 8 * k4, bdesc + 2 * k4, idesc, (kb | k4) != 0 ? 1u : 0u);
          tc_commit(&S.b_empty[sb]);
          tc_commit(&S.a_empty[sa]);
        }
        if (ok) tc_commit(&S.acc_full[b]);
      }
      // All issued MMAs complete before TMEM is released.
      tc_commit(&S.drain);
      mbar_wait(&S.drain, 0, nullptr, p.err, kDevTimeoutDrain, 100000000ull);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ A unpackers: one weight row per thread
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int jobs = my_tiles * p.kblocks;
    uint32_t buf[kUnpackPrefetch][8];
#pragma unroll
    for (int j = 0; j < kUnpackPrefetch; ++j)
      if (j < jobs) unpack_load<kAligned>(p, j, row_in_tile, buf[j]);
    bool ok = true;
    for (int j0 = 0; j0 < jobs && ok; j0 += kUnpackPrefetch) {
#pragma unroll
      for (int jj = 0; jj < kUnpackPrefetch; ++jj) {
        const int j = j0 + jj;
        if (j >= jobs) break;
        const int s = j % kAStages;
        uint32_t v[32];
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
          for (int c = 0; c < 4; ++c) v[4 * w + c] = (buf[jj][w] >> (2 * c)) & 0x03030303u;
        if (j + kUnpackPrefetch < jobs) unpack_load<kAligned>(p, j + kUnpackPrefetch, row_in_tile, buf[jj]);
        if (!warp_wait(&S.a_empty[s], ((j / kAStages) & 1) ^ 1, abort_flag, p.err, kDevTimeoutUnpack)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st_32x32b_x32(lane_base + kACol + 32 * s, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.a_full[s]);
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ epilogue: one weight row per thread
    // Warp 8+e reads TMEM lane quarter e%4 and the 64 token columns of half e/4.
    const int ew = warp - 8;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    double* s_inv = S.tok_inv[ew];
    int32_t* s_rs = S.tok_rs[ew];
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int b = lt & 1;
      const int tile = blockIdx.x + lt * gridDim.x;
      const int m0 = (tile / p.tiles_n) * kBN + 64 * half;
      const int64_t n = (int64_t)(tile % p.tiles_n) * kBM + quarter * 32 + lane;
      const bool nvalid = n < p.N;
      const float dn = nvalid ? __ldg(p.D + n) : 0.0f;
      // Per-token constants of this warp's 64 tokens (two per lane).
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int mm = m0 + 32 * h + lane;
        const bool ok = mm < p.M;
        s_inv[32 * h + lane] = ok ? __drcp_rn((double)__ldg(p.s_x + mm)) : 0.0;
        s_rs[32 * h + lane] = ok ? __ldg(p.rowsum + mm) : 0;
      }
      __syncwarp();
      if (!warp_wait(&S.acc_full[b], (lt >> 1) & 1, abort_flag, p.err, kDevTimeoutEpilogue)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + kAccCol + 128 * b + 64 * half + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * c + j;
          const int m = m0 + t;
          const int a = (int)v[j] - s_rs[t];
          if (m < p.M && nvalid) {
            if (kAccOut)
              p.acc_out[(int64_t)m * p.N + n] = a;
            else
              __stcs(p.y + (int64_t)m * p.N + n, __fmul_rn(div_by_scale(a, s_inv[t]), dn));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[b]);
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
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

template <bool kAligned, bool kAccOut>
static cudaError_t launch_gemm_t(const CUtensorMap& tmap, const GemmParams& p, int grid, cudaStream_t stream) {
  auto kern = gemm_kernel<kAligned, kAccOut>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemLaunch);
  if (e != cudaSuccess) return e;
  kern<<<grid, kGemmThreads, kGemmSmemLaunch, stream>>>(tmap, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                        int32_t* acc_out, void* ws, cudaStream_t stream, int num_sms) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  int8_t* q = reinterpret_cast<int8_t*>(base + ws_q_off(M));
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t gstride[1] = {(cuuint64_t)K};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
  const cuuint32_t estride[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, gdim, gstride, box, estride,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  GemmParams p;
  p.packed = packed;
  p.D = D;
  p.s_x = reinterpret_cast<const float*>(base + ws_sx_off(M));
  p.rowsum = reinterpret_cast<const int32_t*>(base + ws_rowsum_off(M));
  p.y = y;
  p.acc_out = acc_out;
  p.err = reinterpret_cast<uint32_t*>(base);
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.wpr = (int)(K / 16);
  p.kblocks = (int)((K + kBK - 1) / kBK);
  p.tiles_n = (int)((N + kBM - 1) / kBM);
  const int64_t tiles_m = (M + kBN - 1) / kBN;
  const int64_t nt = tiles_m * p.tiles_n;
  if (nt > 0x7FFFFFFF) return cudaErrorInvalidValue;
  p.num_tiles = (int)nt;
  const int grid = (int)(nt < num_sms ? nt : num_sms);
  const bool aligned = (p.wpr % 4) == 0;
  if (acc_out != nullptr)
    return aligned ? launch_gemm_t<true, true>(tmap, p, grid, stream) : launch_gemm_t<false, true>(tmap, p, grid, stream);
  return aligned ? launch_gemm_t<true, false>(tmap, p, grid, stream) : launch_gemm_t<false, false>(tmap, p, grid, stream);
}

}  // namespace bl
