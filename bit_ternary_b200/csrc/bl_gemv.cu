// bl_gemv.cu - decode GEMV (M <= 16 tokens) with ActQuant fused in.
//
// The operation is the BitLinear product of "Core AI model zoo - BitVLA",
// section 2 (M=1 decode, arbitrary K with K % 16 == 0, any N, per-row scale
// D [N,1]), with the wrapper's ActQuant (section 1) done inside the kernel.
//
// Design (B200): the packed weights are the only large stream (2 bits per
// weight), read once with 128-bit coalesced loads. A warp works on a 16-row
// tile; lane (g, t) = (lane/4, lane%4) loads words 4t..4t+3 of a 16-word
// (256-code) unit for rows g and g+8, so the four lanes of a row read 64
// contiguous bytes. Unpacking is one AND per 4 codes: for class c in 0..3,
// word & (0x03030303 << 2c) leaves, in byte b, (code[4b+c]+1) << 2c. Those
// bytes feed mma.sync.m16n8k32 (u8 weights x s8 activations) directly, with
// one accumulator set per class; the classes are recombined exactly as
// acc0 + acc1/4 + acc2/16 + acc3/64 (each accumulator is an exact multiple).
// The activations are quantised per CTA into shared memory in the matching
// order (inside every 16 columns, position 4c+b holds column 4b+c), so the
// B fragments are plain 32-bit shared loads. sum q*(code+1) - sum q gives the
// signed result.
#include "bl_internal.h"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = 8;
constexpr int kRing = 4;  // 256-code units of packed weights in flight per warp

struct GemvParams {
  const float* x;
  const uint32_t* packed;
  const float* D;
  float* y;
  int32_t* acc_out;
  uint32_t* err_reset;
  int M;
  int64_t N;
  int K;
  int wpr;       // packed words per row = K/16
  int n_units;   // ceil(wpr / 16)
  int R;         // 16-row tiles per CTA (1, 2 or 4)
  int q_stride;  // shared bytes per token row
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <bool kAligned>
__device__ __forceinline__ void load_unit(const uint32_t* __restrict__ rowp, bool valid, int w0, int wpr,
                                          uint32_t (&w)[4]) {
  if (kAligned) {
    // wpr % 4 == 0 and w0 % 4 == 0: the four words are all in or all out.
    if (valid && w0 < wpr) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(rowp + w0));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
      w[0] = w[1] = w[2] = w[3] = 0u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = (valid && w0 + j < wpr) ? __ldg(rowp + w0 + j) : 0u;
  }
}

template <int MT, bool kAligned, bool kAccOut>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* sq = smem;                                            // [M][q_stride] permuted int8
  float* s_sx = reinterpret_cast<float*>(smem + p.M * p.q_stride);  // [16]
  int32_t* s_rsum = reinterpret_cast<int32_t*>(s_sx + 16);          // [16]
  uint32_t* s_amax = reinterpret_cast<uint32_t*>(s_rsum + 16);      // [16]
  int32_t* s_red = reinterpret_cast<int32_t*>(s_amax + 16);         // [8][32][4*MT]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int R = p.R;
  const int rt = warp % R, ks = warp / R, nks = kGemvWarps / R;
  const int64_t row0 = ((int64_t)blockIdx.x * R + rt) * 16;
  const int64_t rowA = row0 + g, rowB = row0 + g + 8;
  const bool validA = rowA < p.N, validB = rowB < p.N;
  const uint32_t* rowpA = p.packed + (validA ? rowA : 0) * (int64_t)p.wpr;
  const uint32_t* rowpB = p.packed + (validB ? rowB : 0) * (int64_t)p.wpr;

  // Issue the weight loads of this warp's first kRing units (units ks, ks+nks, ...)
  // before quantising, so their DRAM latency overlaps the ActQuant phase.
  uint32_t wa[kRing][4], wb[kRing][4];
#pragma unroll
  for (int i = 0; i < kRing; ++i) {
    const int u = ks + i * nks;
    load_unit<kAligned>(rowpA, validA && u < p.n_units, u * 16 + 4 * t, p.wpr, wa[i]);
    load_unit<kAligned>(rowpB, validB && u < p.n_units, u * 16 + 4 * t, p.wpr, wb[i]);
  }

  if (p.err_reset != nullptr && blockIdx.x == 0 && tid == 0) *p.err_reset = 0u;
  if (tid < 16) {
    s_amax[tid] = 0u;
    s_rsum[tid] = 0;
  }
  __syncthreads();

  // ---- fused ActQuant: pass 1, max|x| per token (non-negative floats order as uints)
  const int G = p.K >> 4;
  const int total = p.M * G;
  for (int idx = tid; idx < total; idx += kGemvThreads) {
    const int m = idx / G, grp = idx - m * G;
    const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)m * p.K) + 4 * grp;
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = __ldg(xr + j);
      a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    atomicMax(&s_amax[m], __float_as_uint(a));
  }
  __syncthreads();
  // ---- pass 2: quantise into shared memory in the permuted order, row sums
  for (int idx = tid; idx < total; idx += kGemvThreads) {
    const int m = idx / G, grp = idx - m * G;
    const float sx = __fdiv_rn(kQmax, fmaxf(__uint_as_float(s_amax[m]), kFloor));
    const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)m * p.K) + 4 * grp;
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 f = __ldg(xr + j);
      v[4 * j + 0] = quant_i8(f.x, sx);
      v[4 * j + 1] = quant_i8(f.y, sx);
      v[4 * j + 2] = quant_i8(f.z, sx);
      v[4 * j + 3] = quant_i8(f.w, sx);
    }
    uint32_t w4[4];
    int rs = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint32_t word = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) word |= (uint32_t)(v[perm16(4 * r + b)] & 0xFF) << (8 * b);
      w4[r] = word;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) rs += v[j];
    *reinterpret_cast<uint4*>(sq + (int64_t)m * p.q_stride + 16 * grp) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    atomicAdd(&s_rsum[m], rs);
    if (grp == 0) s_sx[m] = sx;
  }
  __syncthreads();

  // ---- main loop over 256-code units
  int acc[4][MT][4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[c][mt][i] = 0;

  for (int base = 0; ks + base * nks < p.n_units; base += kRing) {
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
      const int u = ks + (base + i) * nks;
      if (u >= p.n_units) break;
      uint4 Q[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int tok = g + 8 * mt;
        if (tok < p.M) {
          const uint8_t* qp = sq + (int64_t)tok * p.q_stride + 16 * (u * 16 + 4 * t);
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) Q[mt][i4] = *reinterpret_cast<const uint4*>(qp + 16 * i4);
        } else {
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) Q[mt][i4] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t mask = 0x03030303u << (2 * c);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = wa[i][2 * h] & mask, a2 = wa[i][2 * h + 1] & mask;
          const uint32_t a1 = wb[i][2 * h] & mask, a3 = wb[i][2 * h + 1] & mask;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint4& q0 = Q[mt][2 * h];
            const uint4& q1 = Q[mt][2 * h + 1];
            const uint32_t b0 = c == 0 ? q0.x : (c == 1 ? q0.y : (c == 2 ? q0.z : q0.w));
            const uint32_t b1 = c == 0 ? q1.x : (c == 1 ? q1.y : (c == 2 ? q1.z : q1.w));
            mma_u8s8(acc[c][mt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      // Refill this ring slot with the unit kRing positions further on.
      const int un = u + kRing * nks;
      load_unit<kAligned>(rowpA, validA && un < p.n_units, un * 16 + 4 * t, p.wpr, wa[i]);
      load_unit<kAligned>(rowpB, validB && un < p.n_units, un * 16 + 4 * t, p.wpr, wb[i]);
    }
  }

  // ---- recombine the four classes (exact) and reduce over the K-split warps
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = acc[0][mt][i] + (acc[1][mt][i] >> 2) + (acc[2][mt][i] >> 4) + (acc[3][mt][i] >> 6);
      s_red[(warp * 32 + lane) * (4 * MT) + mt * 4 + i] = r;
    }
  __syncthreads();

  const int rows_cta = 16 * R;
  const int outs = rows_cta * p.M;
  for (int idx = tid; idx < outs; idx += kGemvThreads) {
    const int tok = idx / rows_cta;
    const int rr = idx - tok * rows_cta;
    const int rt2 = rr >> 4, r16 = rr & 15;
    const int64_t row = ((int64_t)blockIdx.x * R + rt2) * 16 + r16;
    if (row >= p.N) continue;
    const int gg = r16 & 7, half = r16 >> 3;
    const int mt = tok >> 3, col = tok & 7;
    const int ln = gg * 4 + (col >> 1);
    const int reg = mt * 4 + half * 2 + (col & 1);
    int sum = 0;
    for (int k2 = 0; k2 < nks; ++k2) sum += s_red[((rt2 + R * k2) * 32 + ln) * (4 * MT) + reg];
    const int a = sum - s_rsum[tok];
    if (kAccOut)
      p.acc_out[(int64_t)tok * p.N + row] = a;
    else
      p.y[(int64_t)tok * p.N + row] = rescale(a, s_sx[tok], __ldg(p.D + row));
  }
}

template <int MT, bool kAligned, bool kAccOut>
static cudaError_t launch_gemv_t(const GemvParams& p, int grid, size_t smem, cudaStream_t stream) {
  auto kern = gemv_kernel<MT, kAligned, kAccOut>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, kGemvThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                        const float* D, float* y, int32_t* acc_out, uint32_t* err_reset, cudaStream_t stream,
                        int num_sms) {
  GemvParams p;
  p.err_reset = err_reset;
  p.x = x;
  p.packed = packed;
  p.D = D;
  p.y = y;
  p.acc_out = acc_out;
  p.M = (int)M;
  p.N = N;
  p.K = (int)K;
  p.wpr = (int)(K / 16);
  p.n_units = (p.wpr + 15) / 16;
  p.q_stride = (int)gemv_q_stride(K);
  // Rows per CTA: as many 16-row tiles as keep every warp within kRing units
  // (so all of its loads are in flight at once) while the grid still covers
  // every SM; more rows per CTA amortise the per-CTA quantisation of x.
  const int64_t tiles = (N + 15) / 16;
  p.R = 1;
  for (int r : {4, 2}) {
    const int units_per_warp = (p.n_units * r + kGemvWarps - 1) / kGemvWarps;
    if (units_per_warp <= kRing && (tiles + r - 1) / r >= num_sms) {
      p.R = r;
      break;
    }
  }
  const int64_t grid = (tiles + p.R - 1) / p.R;
  const int MT = M <= 8 ? 1 : 2;
  const size_t smem = (size_t)M * p.q_stride + 3 * 16 * 4 + (size_t)kGemvWarps * 32 * 4 * MT * 4;
  const bool aligned = (p.wpr % 4) == 0;
  const bool accout = acc_out != nullptr;
#define BL_GEMV_CASE(MT_, AL_, AO_) \
  if (MT == MT_ && aligned == AL_ && accout == AO_) return launch_gemv_t<MT_, AL_, AO_>(p, (int)grid, smem, stream);
  BL_GEMV_CASE(1, true, false)
  BL_GEMV_CASE(1, false, false)
  BL_GEMV_CASE(2, true, false)
  BL_GEMV_CASE(2, false, false)
  BL_GEMV_CASE(1, true, true)
  BL_GEMV_CASE(1, false, true)
  BL_GEMV_CASE(2, true, true)
  BL_GEMV_CASE(2, false, true)
#undef BL_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace bl
