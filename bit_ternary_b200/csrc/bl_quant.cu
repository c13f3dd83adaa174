// bl_quant.cu - WeightQuant + 2-bit pack and per-token ActQuant kernels.
//
// WeightQuant ("Core AI model zoo - BitVLA", section 1; "BitNet-Embeddings
// I2_S guide", section 3.3): s = 1/mean(|W|), code = round(W*s).clamp(-1,1),
// stored as code+1, 16 codes per 32-bit word (BitVLA page, section 2).
// ActQuant (BitVLA page, section 1): per token, round(x*127/max|x|)
// clamped to int8.
//
// The mean of |W| must be identical however the reduction is ordered: it is
// the exact mean, correctly rounded to fp32 once. A first pass sums |w| in
// fp64 with a known bound on its rounding error; when the two fp32 roundings
// of the bounds agree, that is the correctly rounded mean. Otherwise (an fp32
// rounding boundary within ~2^-44 of the mean) the exact path runs: every
// |w| = m * 2^(max(e,1)-150), the 24-bit significands m are summed, in
// integers, into bins by weight (exact and order independent), and a single
// thread forms the exact total and divides it by N*K with one correct rounding.
#include "bl_internal.h"

namespace bl {

// ------------------------------------------------------------------ pack --
constexpr int kBinThreads = 256;
constexpr int kBinWarps = kBinThreads / 32;
constexpr int kWindow = 38;  // binades below a batch's largest exponent summed in one 64-bit word

// Exact per-weight sums of the significands of |W|. |w| = m * 2^(ee-1) units
// of 2^-149, with m < 2^24 and ee = max(biased exponent, 1). A warp takes 128
// weights at a time (one float4 per lane) and the batch's largest ee, E; each
// lane adds m << (ee - base) for base = max(E - kWindow, 1) into a 64-bit word
// (4 terms below 2^62 each), the warp sums that word in three 21-bit chunks
// (each chunk sum < 2^27) and lane 0 adds them to the bins base, base+21 and
// base+42 of a per-warp shared copy. Weights below the window go to their own
// bin. Every step is integer arithmetic, so the result does not depend on the
// order of the reduction.
// Run by one CTA of kBinThreads threads over every float4 of W (the rare
// case where the fp64 pass cannot decide); sbins is its shared scratch.
template <bool kBf16>
__device__ void absum_bins_block(const void* __restrict__ W, int64_t n4, unsigned long long* __restrict__ bins,
                                 unsigned long long (*sbins)[kPackBins]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kBinWarps * kPackBins; i += blockDim.x) (&sbins[0][0])[i] = 0ull;
  __syncthreads();
  unsigned long long* my = sbins[warp];
  const int64_t stride = (int64_t)blockDim.x;
  // Warp-uniform loop bound: every lane reaches the warp reductions.
  const int64_t base0 = (int64_t)(threadIdx.x & ~31);
  for (int64_t wb = base0; wb < n4; wb += stride) {
    const int64_t i = wb + lane;
    uint32_t m[4], ee[4];
    uint32_t emax = 0u, nonfinite = 0u;
    if (i < n4) {
      const float4 v = load4<kBf16>(W, i);
      const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t b = __float_as_uint(vals[j]) & 0x7FFFFFFFu;
        const uint32_t e = b >> 23;
        m[j] = (b & 0x7FFFFFu) | (e != 0 ? 0x800000u : 0u);
        ee[j] = e > 1 ? e : 1;
        if (e == 255) {
          nonfinite = 1u;
          m[j] = 0u;
        }
        if (m[j] != 0u && ee[j] > emax) emax = ee[j];
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) m[j] = 0u, ee[j] = 1u;
    }
    const uint32_t E = __reduce_max_sync(0xFFFFFFFFu, emax);
    const uint32_t base = E > (uint32_t)kWindow + 1u ? E - (uint32_t)kWindow : 1u;
    unsigned long long acc = 0ull;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (m[j] == 0u) continue;
      if (ee[j] >= base)
        acc += (unsigned long long)m[j] << (ee[j] - base);
      else
        atomicAdd(&my[ee[j]], (unsigned long long)m[j]);  // more than kWindow binades below the batch maximum
    }
    const uint32_t c0 = __reduce_add_sync(0xFFFFFFFFu, (uint32_t)(acc & 0x1FFFFFull));
    const uint32_t c1 = __reduce_add_sync(0xFFFFFFFFu, (uint32_t)((acc >> 21) & 0x1FFFFFull));
    const uint32_t c2 = __reduce_add_sync(0xFFFFFFFFu, (uint32_t)(acc >> 42));
    const uint32_t nf = __reduce_add_sync(0xFFFFFFFFu, nonfinite);
    if (lane == 0) {
      if (c0) atomicAdd(&my[base], (unsigned long long)c0);
      if (c1) atomicAdd(&my[base + 21], (unsigned long long)c1);
      if (c2) atomicAdd(&my[base + 42], (unsigned long long)c2);
      if (nf) atomicAdd(&my[kPackNonFiniteBin], (unsigned long long)nf);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kPackBins; e += blockDim.x) {
    unsigned long long s = 0;
#pragma unroll
    for (int w = 0; w < kBinWarps; ++w) s += sbins[w][e];
    if (s) atomicAdd(&bins[e], s);
  }
  __syncthreads();
}

// Correctly rounded fp32 of S * 2^-149 / n, where S = sum_e bins[e] * 2^(max(e,1)-1).
// Results below the normal range are returned as 0 (they lie far below the
// 1e-5 floor that is applied afterwards). One thread. n = N*K < 2^48 (N < 2^31,
// K <= 2^17), and a tensor that fits in device memory has n < 2^36, so every
// bin is below 2^60 and S below 2^313.
__device__ void absmean_exact_block(const unsigned long long* __restrict__ gbins, uint64_t n,
                                    float* __restrict__ scal, uint32_t* __restrict__ status) {
  // S = sum_e bins[e] * 2^(max(e,1)-1) as 11 little-endian 32-bit limbs (used
  // bins < 2^60 at indices <= 258: S < 2^318). The block adds every bin's
  // (up to three) limb parts into 64-bit per-limb sums with shared atomics
  // (at most ~260 parts of < 2^32 per limb: no overflow); one thread then
  // propagates the carries and divides.
  constexpr int L = 11;
  __shared__ unsigned long long bins[kPackBins];
  __shared__ unsigned long long limb_sum[L + 3];
  __shared__ uint32_t sS[L];
  for (int i = threadIdx.x; i < kPackBins; i += blockDim.x) bins[i] = gbins[i];
  for (int i = threadIdx.x; i < L + 3; i += blockDim.x) limb_sum[i] = 0ull;
  __syncthreads();
  const bool nonfinite = bins[kPackNonFiniteBin] != 0ull;
  if (!nonfinite) {
    for (int e = threadIdx.x; e < kPackNonFiniteBin; e += blockDim.x) {
      const unsigned long long v = bins[e];
      if (v == 0ull) continue;
      const int sh = (e > 1 ? e : 1) - 1;
      const int limb = sh >> 5, bit = sh & 31;
      // v << bit spans up to three limbs.
      const uint32_t p0 = (uint32_t)(v << bit);
      const uint32_t p1 = bit == 0 ? (uint32_t)(v >> 32) : (uint32_t)(v >> (32 - bit));
      const uint32_t p2 = bit == 0 ? 0u : (uint32_t)((v >> 32) >> (32 - bit));
      atomicAdd(&limb_sum[limb], (unsigned long long)p0);
      atomicAdd(&limb_sum[limb + 1], (unsigned long long)p1);
      if (p2 != 0u) atomicAdd(&limb_sum[limb + 2], (unsigned long long)p2);
    }
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (nonfinite) {
    *status = 1u;  // non-finite input
    scal[0] = __int_as_float(0x7FC00000);
    scal[1] = __int_as_float(0x7FC00000);
    return;
  }
  {
    unsigned long long carry = 0ull;
#pragma unroll
    for (int i = 0; i < L; ++i) {
      const unsigned long long t = limb_sum[i] + carry;
      sS[i] = (uint32_t)t;
      carry = t >> 32;
    }
  }
  // Long division of S * 2^F by n (n < 2^48), 16-bit digits MSB first: the
  // remainder stays below n, so remainder * 2^16 + digit fits in 64 bits.
  // Digit d covers bits [32L + F - 16(d+1), +16) of S * 2^F.
  constexpr int F = 32;
  constexpr int kDigits = (32 * L + F) / 16;  // 24
  auto digit = [&](int d) -> uint32_t {
    const int bit = 32 * L + F - 16 * (d + 1);
    if (bit < F) return 0u;
    const int j = bit - F;
    return (sS[j >> 5] >> (j & 31)) & 0xFFFFu;
  };
  // Leading zero digits of S * 2^F give zero quotient digits and leave the
  // remainder at 0. From the first nonzero quotient digit on, four digits
  // hold the leading 24 bits, the round bit and the start of the sticky bits;
  // every bit below them is nonzero exactly when the remainder or a digit of
  // S * 2^F not yet taken is.
  int d = 0;
  while (d < kDigits && digit(d) == 0u) ++d;
  unsigned long long rem = 0ull, w = 0ull;
  uint32_t q_lead = 0u;
  int dl = -1, got = 0;
  for (; d < kDigits && got < 4; ++d) {
    const unsigned long long cur = (rem << 16) | digit(d);
    const uint32_t qd = (uint32_t)(cur / n);
    rem = cur % n;
    if (dl < 0 && qd != 0u) {
      dl = d;
      q_lead = qd;
    }
    if (dl >= 0) {
      w = (w << 16) | qd;
      ++got;
    }
  }
  bool rest = rem != 0ull;
  for (int dd = d; dd < kDigits && !rest; ++dd) rest = digit(dd) != 0u;
  float mean = 0.0f;
  if (dl >= 0) {
    w <<= 16 * (4 - got);                                 // digits past the last one are zero
    const int lb = 31 - __clz(q_lead);                    // leading bit inside digit dl
    const int lead = 16 * (kDigits - 1 - dl) + lb;        // its index from the quotient's LSB
    if (lead >= 24) {
      const int top = 48 + lb;                            // the leading bit's index in w
      uint32_t sig = (uint32_t)(w >> (top - 23)) & 0xFFFFFFu;
      const uint32_t round_bit = (uint32_t)(w >> (top - 24)) & 1u;
      const uint32_t sticky = (rest || (w & ((1ull << (top - 24)) - 1ull)) != 0ull) ? 1u : 0u;
      int E = lead - 149 - F;  // value = 1.xxx * 2^E
      if (round_bit && (sticky || (sig & 1u))) {
        ++sig;
        if (sig == (1u << 24)) {
          sig >>= 1;
          ++E;
        }
      }
      if (E >= -126 && E <= 127) mean = __uint_as_float(((uint32_t)(E + 127) << 23) | (sig & 0x7FFFFFu));
    }
  }
  const float mean_c = fmaxf(mean, kFloor);
  scal[0] = mean_c;
  scal[1] = __fdiv_rn(1.0f, mean_c);
  *status = 0u;
}

// First pass: fp64 sums of |w|. Each thread adds its weights in sequence
// (four float4 loads in flight), then the warp (butterfly, 5 levels) and the
// CTA (8 warps, 3 levels) add in a fixed order; one partial per CTA. Each |w|
// is exact in fp64. The last CTA to finish adds the partials in a fixed order
// and decides the mean: the sum S has gone through at most `depth` roundings
// on any path from a weight (a bound the host derives from the launch shape),
// so with non-negative terms the exact sum lies within S * depth * 2^-52 of S
// (twice the first-order bound). If the fp32 roundings of the two ends of that
// interval, divided by n with directed rounding, agree, that is the correctly
// rounded mean. Otherwise the same CTA runs the exact integer path over all of
// W (slow, and reached only within ~2^-44 of a rounding boundary).
constexpr int kSumThreads = kBinThreads;
constexpr int kSumUnroll = 4;
template <bool kBf16>
__global__ void __launch_bounds__(kSumThreads) absum_f64_kernel(const void* __restrict__ W, int64_t n4, uint64_t n,
                                                                int depth, double* __restrict__ partial,
                                                                unsigned long long* __restrict__ bins,
                                                                uint32_t* __restrict__ done,
                                                                float* __restrict__ scal,
                                                                uint32_t* __restrict__ status,
                                                                uint32_t* __restrict__ sticky) {
  __shared__ double red[kSumThreads / 32];
  __shared__ int is_last;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double s = 0.0;
  uint32_t bad = 0u;
  for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < n4; i0 += kSumUnroll * stride) {
    float4 v[kSumUnroll];
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = i < n4 ? load4<kBf16>(W, i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u) {
      const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bad |= (__float_as_uint(f[j]) & 0x7F800000u) == 0x7F800000u;
        s += (double)fabsf(f[j]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) red[warp] = s;
  if (__any_sync(0xFFFFFFFFu, bad != 0u) && lane == 0) atomicAdd(&bins[kPackNonFiniteBin], 1ull);
  __syncthreads();
  if (threadIdx.x == 0) {
    const double t0 = red[0] + red[1], t1 = red[2] + red[3], t2 = red[4] + red[5], t3 = red[6] + red[7];
    partial[blockIdx.x] = (t0 + t1) + (t2 + t3);
    __threadfence();
    is_last = atomicAdd(done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // The last CTA: every partial and non-finite count is visible.
  const volatile double* vp = partial;
  s = 0.0;
  for (int i = threadIdx.x; i < (int)gridDim.x; i += blockDim.x) s += vp[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  __syncthreads();  // every warp has read red[] above
  if (lane == 0) red[warp] = s;
  __syncthreads();
  const bool nonfinite = *reinterpret_cast<volatile unsigned long long*>(&bins[kPackNonFiniteBin]) != 0ull;
  if (nonfinite) {
    if (threadIdx.x == 0) {
      *status = 1u;  // non-finite input: this call writes neither packed nor D
      atomicOr(sticky, 1u);
      scal[0] = __int_as_float(0x7FC00000);
      scal[1] = __int_as_float(0x7FC00000);
    }
    return;
  }
  const double t0 = red[0] + red[1], t1 = red[2] + red[3], t2 = red[4] + red[5], t3 = red[6] + red[7];
  const double S = (t0 + t1) + (t2 + t3);
  const double rel = (double)depth * 0x1p-52;
  const double lo = __ddiv_rd(__dmul_rd(S, 1.0 - rel), (double)n);
  const double hi = __ddiv_ru(__dmul_ru(S, 1.0 + rel), (double)n);
  const float c1 = __double2float_rn(lo), c2 = __double2float_rn(hi);
  if (c1 == c2) {  // uniform over the CTA: every thread computed the same values
    if (threadIdx.x == 0) {
      // Below the normal range the exact path gives 0; either way the floor applies.
      const float mean_c = fmaxf(c1, kFloor);
      scal[0] = mean_c;
      scal[1] = __fdiv_rn(1.0f, mean_c);
      *status = 0u;
    }
    return;
  }
  __shared__ unsigned long long sbins[kBinWarps][kPackBins];
  absum_bins_block<kBf16>(W, n4, bins, sbins);
  absmean_exact_block(bins, n, scal, status);
}

// Each thread ternarises one float4 (4 codes = one byte of a packed word);
// lanes 4j..4j+3 of a warp hold the four bytes of one word and combine them
// with shuffles. Also writes D[n] = mean_c. Warps take 32-float4 chunks from
// the end of W backwards: the first pass read W from the start, so its tail
// is what the L2 still holds.
template <bool kBf16>
__global__ void __launch_bounds__(256) ternarize_pack_kernel(const void* __restrict__ W, int64_t n4,
                                                             const float* __restrict__ scal,
                                                             const uint32_t* __restrict__ status,
                                                             uint32_t* __restrict__ packed, float* __restrict__ D,
                                                             int64_t N) {
  if (*status != 0u) return;
  const float mean_c = scal[0];
  const float s = scal[1];
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // Loop bound is warp-uniform so every lane reaches the shuffles. Two chunks
  // per iteration, both loads issued before either is used.
  const int64_t nchunks = (n4 + 31) >> 5;
  const int64_t cstride = stride >> 5;
  for (int64_t c = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; c < nchunks; c += 2 * cstride) {
    int64_t i[2];
    float4 v[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t ch = c + h * cstride;
      i[h] = ch < nchunks ? ((nchunks - 1 - ch) << 5) + lane : n4;
      v[h] = i[h] < n4 ? load4<kBf16>(W, i[h]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t byte = code_plus_one(v[h].x, s) | (code_plus_one(v[h].y, s) << 2) |
                            (code_plus_one(v[h].z, s) << 4) | (code_plus_one(v[h].w, s) << 6);
      uint32_t word = byte << (8 * (lane & 3));
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
      if ((lane & 3) == 0 && i[h] < n4) packed[i[h] >> 2] = word;
    }
  }
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += stride) D[n] = mean_c;
}

// -------------------------------------------------------------- ActQuant --
// One CTA per token row. Pass 1: max|x| (exact). Pass 2: quantise 16 columns
// per thread-iteration and store them as one 16-byte vector, in natural
// column order or in the kernel-private order perm16 (see bl_device.cuh).
template <bool kPerm, bool kBf16>
__global__ void __launch_bounds__(256) act_quant_kernel(const void* __restrict__ x, int64_t K,
                                                        int8_t* __restrict__ q, float* __restrict__ s_out,
                                                        int32_t* __restrict__ rowsum_out,
                                                        uint32_t* __restrict__ err_reset) {
  // A decode launch that waits on these codes may start streaming its weights.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (err_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_reset = 0u;
  __shared__ float red_f[8];
  __shared__ int red_i[8];
  const int64_t m = blockIdx.x;
  const int64_t xr = m * (K >> 2);  // first float4 (group of 4 elements) of the row
  const int ngroups = (int)(K >> 4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;

  float amax = 0.0f;
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = load4<kBf16>(x, xr + 4 * g + j);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) red_f[warp] = amax;
  __syncthreads();
  amax = 0.0f;
  for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, red_f[w]);
  const float sx = __fdiv_rn(kQmax, fmaxf(amax, kFloor));

  int rsum = 0;
  int8_t* qr = q + m * K;
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 f = load4<kBf16>(x, xr + 4 * g + j);
      v[4 * j + 0] = quant_code(f.x, sx);
      v[4 * j + 1] = quant_code(f.y, sx);
      v[4 * j + 2] = quant_code(f.z, sx);
      v[4 * j + 3] = quant_code(f.w, sx);
    }
    uint32_t w4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint32_t word = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int p = 4 * r + b;
        const int src = kPerm ? perm16(p) : p;
        word |= (uint32_t)(v[src] & 0xFF) << (8 * b);
      }
      w4[r] = word;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) rsum += v[j];
    *reinterpret_cast<uint4*>(qr + 16 * (int64_t)g) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xFFFFFFFFu, rsum, o);
  if (lane == 0) red_i[warp] = rsum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < nwarps; ++w) t += red_i[w];
    s_out[m] = sx;
    if (rowsum_out != nullptr) rowsum_out[m] = t;
  }
}

// ------------------------------------------------------ wait self-test --
// One thread waits on a barrier that is never completed; the bounded wait must
// give up after limit_ns and record kDevTimeoutSelftest in the error word.
__global__ void selftest_wait_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait(&bar, 0, &abort_flag, err, kDevTimeoutSelftest, limit_ns);
}

cudaError_t launch_selftest_wait(uint32_t* err, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

// Register-resident variant for rows of up to 256 * 16 * kG columns: each
// thread loads its kG groups of 16 values once, the block reduces max|x|, and
// the same registers are quantised and stored (one read of x, one write of q).
// ActQuant with one warp per token, for rows of up to 32 * kWG groups of 16
// columns (K <= 3072): every lane keeps its groups in registers (up to 24
// 16-byte loads in flight), max|x| and the row sum are warp reductions, and no
// block barrier is needed. The same arithmetic as act_quant_reg_kernel.
template <bool kPerm, int kWG, bool kBf16>
__global__ void __launch_bounds__(256) act_quant_warp_kernel(const void* __restrict__ x, int64_t M, int64_t K,
                                                             int8_t* __restrict__ q, float* __restrict__ s_out,
                                                             int32_t* __restrict__ rowsum_out,
                                                             uint32_t* __restrict__ err_reset) {
  // A decode launch that waits on these codes may start streaming its weights.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (err_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_reset = 0u;
  const int lane = threadIdx.x & 31;
  const int ngroups = (int)(K >> 4);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t m = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M; m += nwarps) {
    const int64_t xr = m * (K >> 2);
    float4 f[kWG][4];
#pragma unroll
    for (int i = 0; i < kWG; ++i) {
      const int gi = lane + 32 * i;
#pragma unroll
      for (int j = 0; j < 4; ++j) f[i][j] = gi < ngroups ? load4<kBf16>(x, xr + 4 * gi + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kWG; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[i][j].x), fabsf(f[i][j].y)), fmaxf(fabsf(f[i][j].z), fabsf(f[i][j].w))));
    // |x| >= 0, so the order of the bit patterns is the order of the values.
    amax = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax)));
    const float sx = __fdiv_rn(kQmax, fmaxf(amax, kFloor));
    int rsum = 0;
    int8_t* qr = q + m * K;
#pragma unroll
    for (int i = 0; i < kWG; ++i) {
      const int gi = lane + 32 * i;
      if (gi >= ngroups) continue;
      int v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[4 * j + 0] = quant_code(f[i][j].x, sx);
        v[4 * j + 1] = quant_code(f[i][j].y, sx);
        v[4 * j + 2] = quant_code(f[i][j].z, sx);
        v[4 * j + 3] = quant_code(f[i][j].w, sx);
      }
      uint32_t w4[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        uint32_t word = 0u;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int pp = 4 * r + b;
          word |= (uint32_t)(v[kPerm ? perm16(pp) : pp] & 0xFF) << (8 * b);
        }
        w4[r] = word;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) rsum += v[j];
      *reinterpret_cast<uint4*>(qr + 16 * (int64_t)gi) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    rsum = __reduce_add_sync(0xFFFFFFFFu, rsum);
    if (lane == 0) {
      s_out[m] = sx;
      if (rowsum_out != nullptr) rowsum_out[m] = rsum;
    }
  }
}

template <bool kPerm, int kG, bool kBf16>
__global__ void __launch_bounds__(256) act_quant_reg_kernel(const void* __restrict__ x, int64_t K,
                                                            int8_t* __restrict__ q, float* __restrict__ s_out,
                                                            int32_t* __restrict__ rowsum_out,
                                                            uint32_t* __restrict__ err_reset) {
  // A decode launch that waits on these codes may start streaming its weights.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float red_f[8];
  if (err_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_reset = 0u;
  const int64_t m = blockIdx.x;
  const int64_t xr = m * (K >> 2);  // first float4 (group of 4 elements) of the row
  // Cleared before the block barrier below; the warps add their sums after it.
  if (rowsum_out != nullptr && threadIdx.x == 0) rowsum_out[m] = 0;
  const int ngroups = (int)(K >> 4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  float4 f[kG][4];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const int g = threadIdx.x + i * blockDim.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (g < ngroups) f[i][j] = load4<kBf16>(x, xr + 4 * g + j);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[i][j].x), fabsf(f[i][j].y)), fmaxf(fabsf(f[i][j].z), fabsf(f[i][j].w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) red_f[warp] = amax;
  __syncthreads();
  amax = 0.0f;
  for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, red_f[w]);
  const float sx = __fdiv_rn(kQmax, fmaxf(amax, kFloor));
  int rsum = 0;
  int8_t* qr = q + m * K;
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const int g = threadIdx.x + i * blockDim.x;
    if (g >= ngroups) continue;
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[4 * j + 0] = quant_code(f[i][j].x, sx);
      v[4 * j + 1] = quant_code(f[i][j].y, sx);
      v[4 * j + 2] = quant_code(f[i][j].z, sx);
      v[4 * j + 3] = quant_code(f[i][j].w, sx);
    }
    uint32_t w4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint32_t word = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int p = 4 * r + b;
        word |= (uint32_t)(v[kPerm ? perm16(p) : p] & 0xFF) << (8 * b);
      }
      w4[r] = word;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) rsum += v[j];
    *reinterpret_cast<uint4*>(qr + 16 * (int64_t)g) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  if (threadIdx.x == 0) s_out[m] = sx;
  if (rowsum_out != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xFFFFFFFFu, rsum, o);
    if (lane == 0) atomicAdd(rowsum_out + m, rsum);
  }
}

// ------------------------------------------------------ RMSNorm + ActQuant --
// Per-projection RMSNorm before ActQuant ("BitNet-Embeddings I2_S guide",
// section 3.1; rms_norm_eps 1e-6): n = RN(RN(x*r)*g) with
// r = RN(1/RN(sqrt(RN(ms + eps)))) and ms = mean(x^2) correctly rounded once
// from the exact sum. One CTA per token, x and g held in registers; the row
// sum goes out by one atomic per warp onto a word that thread 0 cleared before
// the first block barrier.
//
// ms: each x^2 is exact in fp64, so the fp64 sum S' of the K squares, in any
// order, is within gamma_(K-1) = (K-1)u/(1-(K-1)u) of the exact S (u = 2^-53,
// all terms >= 0), and q = RN64(S'/K) adds one more u. Thread 0 widens q by
// (K+8)*2^-52 in both directions with directed rounding; if both ends round to
// the same fp32, that is RN32(S/K). Otherwise (a rounding boundary inside the
// interval: a few tokens in a million) the block sums the squares exactly in
// integers and divides by K.
template <bool kPerm, int kG>
__global__ void __launch_bounds__(256, kG == 1 ? 3 : (kG == 2 ? 4 : 1)) rms_act_quant_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                            float eps, int64_t K, int8_t* __restrict__ q,
                                                            float* __restrict__ s_out, int32_t* __restrict__ rowsum_out,
                                                            uint32_t* __restrict__ err_reset, int64_t M) {
  __shared__ double red_d[8];
  __shared__ float red_f[8];
  __shared__ float s_ms;
  __shared__ int s_exact;
  __shared__ unsigned long long bins[kRmsBins];
  if (err_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_reset = 0u;
  const int ngroups = (int)(K >> 4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  // A CTA walks tokens blockIdx.x, blockIdx.x + gridDim.x, ... With one
  // 16-column group per thread (kG == 1) the next token's row is loaded into
  // registers while the current one is normalised and quantised, so the row
  // loads of successive tokens overlap the per-token reductions and barriers,
  // and g (the same for every token) is loaded once. Wider rows launch one
  // CTA per token (a second row copy would cost occupancy).
  constexpr bool kGEarly = kG == 1;
  constexpr bool kPrefetch = kG == 1;
  float4 fn[kPrefetch ? kG : 1][4];  // the next token's row (prefetch form only)
  float4 gw[kGEarly ? kG : 1][4];
  auto load_row = [&](int64_t mm, float4 (&dst)[kG][4]) {
    const int64_t xr = mm * (K >> 2);
#pragma unroll
    for (int i = 0; i < kG; ++i) {
      const int gi = threadIdx.x + i * blockDim.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        dst[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (gi < ngroups) dst[i][j] = __ldg(reinterpret_cast<const float4*>(x) + xr + 4 * gi + j);
      }
    }
  };
  if (kGEarly) {
#pragma unroll
    for (int i = 0; i < kG; ++i) {
      const int gi = threadIdx.x + i * blockDim.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        gw[kGEarly ? i : 0][j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (gi < ngroups) gw[kGEarly ? i : 0][j] = __ldg(reinterpret_cast<const float4*>(g) + 4 * gi + j);
      }
    }
  }
  if constexpr (kPrefetch) {
    if ((int64_t)blockIdx.x < M) load_row(blockIdx.x, fn);
  }
#pragma unroll 1
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
  float4 f[kG][4];
  if constexpr (kPrefetch) {
#pragma unroll
    for (int i = 0; i < kG; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) f[i][j] = fn[i][j];
    if (m + gridDim.x < M) load_row(m + gridDim.x, fn);
  } else {
    load_row(m, f);
  }
  // Cleared before the first block barrier; the warps add their sums at the end.
  if (rowsum_out != nullptr && threadIdx.x == 0) rowsum_out[m] = 0;
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < kG; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ss += (double)f[i][j].x * f[i][j].x + (double)f[i][j].y * f[i][j].y;
      ss += (double)f[i][j].z * f[i][j].z + (double)f[i][j].w * f[i][j].w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if (lane == 0) red_d[warp] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double S = 0.0;
    for (int w = 0; w < nwarps; ++w) S += red_d[w];
    const double qd = S / (double)K;
    const double d = (double)(K + 8) * 2.220446049250313e-16;  // (K+8) * 2^-52
    const float flo = __double2float_rn(__dmul_rd(qd, 1.0 - d));
    const float fhi = __double2float_rn(__dmul_ru(qd, 1.0 + d));
    s_exact = flo != fhi;
    s_ms = flo;
  }
  __syncthreads();
  if (s_exact) {  // block-uniform
    for (int b = threadIdx.x; b < kRmsBins; b += blockDim.x) bins[b] = 0ull;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kG; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rms_bins_add(bins, f[i][j].x);
        rms_bins_add(bins, f[i][j].y);
        rms_bins_add(bins, f[i][j].z);
        rms_bins_add(bins, f[i][j].w);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) s_ms = mean_square_exact_f32(bins, (uint32_t)K);
    __syncthreads();
  }
  const float ms = s_ms;
  const float rr = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const int gi = threadIdx.x + i * blockDim.x;
    if (gi >= ngroups) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 gv = kGEarly ? gw[kGEarly ? i : 0][j] : __ldg(reinterpret_cast<const float4*>(g) + 4 * gi + j);
      f[i][j].x = __fmul_rn(__fmul_rn(f[i][j].x, rr), gv.x);
      f[i][j].y = __fmul_rn(__fmul_rn(f[i][j].y, rr), gv.y);
      f[i][j].z = __fmul_rn(__fmul_rn(f[i][j].z, rr), gv.z);
      f[i][j].w = __fmul_rn(__fmul_rn(f[i][j].w, rr), gv.w);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[i][j].x), fabsf(f[i][j].y)), fmaxf(fabsf(f[i][j].z), fabsf(f[i][j].w))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) red_f[warp] = amax;
  __syncthreads();
  amax = 0.0f;
  for (int w = 0; w < nwarps; ++w) amax = fmaxf(amax, red_f[w]);
  const float sx = __fdiv_rn(kQmax, fmaxf(amax, kFloor));
  int rsum = 0;
  int8_t* qr = q + m * K;
#pragma unroll
  for (int i = 0; i < kG; ++i) {
    const int gi = threadIdx.x + i * blockDim.x;
    if (gi >= ngroups) continue;
    int v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[4 * j + 0] = quant_code(f[i][j].x, sx);
      v[4 * j + 1] = quant_code(f[i][j].y, sx);
      v[4 * j + 2] = quant_code(f[i][j].z, sx);
      v[4 * j + 3] = quant_code(f[i][j].w, sx);
    }
    uint32_t w4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint32_t word = 0u;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int p = 4 * r + b;
        word |= (uint32_t)(v[kPerm ? perm16(p) : p] & 0xFF) << (8 * b);
      }
      w4[r] = word;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) rsum += v[j];
    *reinterpret_cast<uint4*>(qr + 16 * (int64_t)gi) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  if (threadIdx.x == 0) s_out[m] = sx;
  if (rowsum_out != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xFFFFFFFFu, rsum, o);
    if (lane == 0) atomicAdd(rowsum_out + m, rsum);
  }
  }  // token loop
}

// ------------------------------------------------------------ launchers --
cudaError_t launch_pack(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                        bool clear_sticky, cudaStream_t stream, int num_sms) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* sticky = reinterpret_cast<uint32_t*>(base);     // OR of every call's failure since the last read
  uint32_t* status = reinterpret_cast<uint32_t*>(base + 4);  // this call's
  uint32_t* done = reinterpret_cast<uint32_t*>(base + 8);  // CTAs of the fp64 pass that have finished
  float* scal = reinterpret_cast<float*>(base + 16);
  unsigned long long* bins = reinterpret_cast<unsigned long long*>(base + kHeaderBytes);
  double* partial = reinterpret_cast<double*>(base + kHeaderBytes + kPackBins * sizeof(unsigned long long));
  const size_t keep = clear_sticky ? 0 : 4;
  cudaError_t err = cudaMemsetAsync(base + keep, 0, kPackWsBytes - keep, stream);
  if (err != cudaSuccess) return err;
  const int64_t n4 = N * K / 4;
  // fp64 pass (and, in its last CTA, the mean): up to 4 CTAs per SM.
  {
    const int64_t want0 = (n4 + kSumThreads * kSumUnroll - 1) / (kSumThreads * kSumUnroll);
    int64_t g0 = want0 < 4 * (int64_t)num_sms ? want0 : 4 * (int64_t)num_sms;
    g0 = g0 < 1 ? 1 : (g0 > kPackSumBlocks ? kPackSumBlocks : g0);
    const int64_t stride = g0 * kSumThreads;
    // Roundings on any path: the thread's sequential adds (4 per float4), the
    // warp's 5 and the CTA's 3 levels, then the last CTA's sequential adds of
    // partials, its warp's 5 and its 3 levels; plus a margin.
    const int64_t per_thread = 4 * ((n4 + stride - 1) / stride);
    const int64_t per_final = (g0 + kSumThreads - 1) / kSumThreads;
    const int depth = (int)(per_thread + 8 + per_final + 8 + 4);
    if (bf16)
      absum_f64_kernel<true><<<(unsigned)g0, kSumThreads, 0, stream>>>(W, n4, (uint64_t)(N * K), depth, partial,
                                                                       bins, done, scal, status, sticky);
    else
      absum_f64_kernel<false><<<(unsigned)g0, kSumThreads, 0, stream>>>(W, n4, (uint64_t)(N * K), depth, partial,
                                                                        bins, done, scal, status, sticky);
  }
  const int64_t want2 = (n4 + 255) / 256;
  const int grid2 = (int)(want2 < 16 * num_sms ? (want2 < 1 ? 1 : want2) : 16 * num_sms);
  if (bf16)
    ternarize_pack_kernel<true><<<grid2, 256, 0, stream>>>(W, n4, scal, status, packed, D, N);
  else
    ternarize_pack_kernel<false><<<grid2, 256, 0, stream>>>(W, n4, scal, status, packed, D, N);
  return cudaGetLastError();
}

// Pre-quantised input: natural-order int8 codes q [M,K] and scales s_x [M]
// (as bitlinear_quant_act writes them) into the forward workspace, in the
// kernel-private column order, with the row sums. One CTA per token; each
// thread moves 16-column groups: byte j of output word r is byte r of input
// word j (the 4x4 byte transpose perm16 describes).
__global__ void __launch_bounds__(256) q_prepare_kernel(const int8_t* __restrict__ q, const float* __restrict__ s_x,
                                                        int64_t K, int8_t* __restrict__ wq, float* __restrict__ wsx,
                                                        int32_t* __restrict__ wrs, uint32_t* __restrict__ err_reset) {
  if (err_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_reset = 0u;
  __shared__ int red[8];
  const int64_t m = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(q + m * K);
  uint4* dst = reinterpret_cast<uint4*>(wq + m * K);
  const int ngroups = (int)(K >> 4);
  int sum = 0;
  for (int g = threadIdx.x; g < ngroups; g += blockDim.x) {
    const uint4 v = __ldg(src + g);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
      o[r] = ((w[0] >> (8 * r)) & 0xFFu) | (((w[1] >> (8 * r)) & 0xFFu) << 8) | (((w[2] >> (8 * r)) & 0xFFu) << 16) |
             (((w[3] >> (8 * r)) & 0xFFu) << 24);
    dst[g] = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int j = 0; j < 4; ++j) sum = __dp4a((int)w[j], 0x01010101, sum);  // sum of the four signed bytes
  }
  sum = __reduce_add_sync(0xFFFFFFFFu, sum);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    wrs[m] = t;
    wsx[m] = s_x[m];
  }
}

cudaError_t launch_q_prepare(const int8_t* q, const float* s_x, int64_t M, int64_t K, int8_t* wq, float* wsx,
                             int32_t* wrs, cudaStream_t stream, uint32_t* err_reset) {
  q_prepare_kernel<<<(unsigned)M, 256, 0, stream>>>(q, s_x, K, wq, wsx, wrs, err_reset);
  return cudaGetLastError();
}

template <bool kBf16>
static cudaError_t launch_act_quant_t(const void* x, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                                      bool permuted, cudaStream_t stream, uint32_t* err_reset) {
  const int64_t ngroups = K / 16;
  // Many tokens with rows of up to 6 groups per lane: one warp per token, no
  // block barrier. A few tokens (decode) keep one CTA per token, which
  // finishes each token sooner (its 16-column groups spread over more warps).
  if (ngroups <= 32 * 6 && M >= 1024) {
    const int wg = (int)((ngroups + 31) / 32);
    const int64_t want = (M + 7) / 8;
    const unsigned grid = (unsigned)(want < 1 ? 1 : (want < 148 * 16 ? want : 148 * 16));
#define BL_AQW(P, G) act_quant_warp_kernel<P, G, kBf16><<<grid, 256, 0, stream>>>(x, M, K, q, s_x, rowsum, err_reset)
#define BL_AQW_G(P)                                                                                         \
  switch (wg) {                                                                                             \
    case 1: BL_AQW(P, 1); break;                                                                            \
    case 2: BL_AQW(P, 2); break;                                                                            \
    case 3: BL_AQW(P, 3); break;                                                                            \
    case 4: BL_AQW(P, 4); break;                                                                            \
    case 5: BL_AQW(P, 5); break;                                                                            \
    default: BL_AQW(P, 6); break;                                                                           \
  }
    if (permuted) {
      BL_AQW_G(true)
    } else {
      BL_AQW_G(false)
    }
#undef BL_AQW_G
#undef BL_AQW
    return cudaGetLastError();
  }
  // Rows of up to 256 threads x 4 groups x 16 values stay in registers.
  int kg = (int)((ngroups + 255) / 256);
  if (kg <= 4) {
    kg = kg <= 1 ? 1 : (kg <= 2 ? 2 : 4);
    int threads = (int)(((ngroups + kg - 1) / kg + 31) / 32 * 32);
    if (threads < 32) threads = 32;
#define BL_AQ(P, G) act_quant_reg_kernel<P, G, kBf16><<<(unsigned)M, threads, 0, stream>>>(x, K, q, s_x, rowsum, err_reset)
    if (permuted) {
      if (kg == 1) BL_AQ(true, 1); else if (kg == 2) BL_AQ(true, 2); else BL_AQ(true, 4);
    } else {
      if (kg == 1) BL_AQ(false, 1); else if (kg == 2) BL_AQ(false, 2); else BL_AQ(false, 4);
    }
#undef BL_AQ
    return cudaGetLastError();
  }
  const int threads = 256;
  // One CTA per token; grids beyond 2^31-1 are rejected by validation.
  if (permuted)
    act_quant_kernel<true, kBf16><<<(unsigned)M, threads, 0, stream>>>(x, K, q, s_x, rowsum, err_reset);
  else
    act_quant_kernel<false, kBf16><<<(unsigned)M, threads, 0, stream>>>(x, K, q, s_x, rowsum, err_reset);
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* x, bool bf16, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                             bool permuted, cudaStream_t stream, uint32_t* err_reset) {
  return bf16 ? launch_act_quant_t<true>(x, M, K, q, s_x, rowsum, permuted, stream, err_reset)
              : launch_act_quant_t<false>(x, M, K, q, s_x, rowsum, permuted, stream, err_reset);
}

}  // namespace bl

namespace bl {

cudaError_t launch_rms_act_quant(const float* x, const float* g, float eps, int64_t M, int64_t K, int8_t* q,
                                 float* s_x, int32_t* rowsum, bool permuted, cudaStream_t stream,
                                 uint32_t* err_reset) {
  const int64_t ngroups = K / 16;
  int kg = (int)((ngroups + 255) / 256);
  if (kg > 4) return cudaErrorInvalidValue;  // K <= 16384
  kg = kg <= 1 ? 1 : (kg <= 2 ? 2 : 4);
  int threads = (int)(((ngroups + kg - 1) / kg + 31) / 32 * 32);
  if (threads < 32) threads = 32;
  // Persistent CTAs (as many as fit, up to one per token), each walking tokens.
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
#define BL_RQ(P, G)                                                                                            \
  do {                                                                                                         \
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rms_act_quant_kernel<P, G>, threads, 0);      \
    if (e != cudaSuccess) return e;                                                                            \
    int64_t grid = (int64_t)sms * (per_sm < 1 ? 1 : per_sm);                                                  \
    if (G > 1 || grid > M) grid = M; /* one CTA per token unless the row prefetch runs */                    \
    rms_act_quant_kernel<P, G><<<(unsigned)grid, threads, 0, stream>>>(x, g, eps, K, q, s_x, rowsum, err_reset, M); \
  } while (0)
  if (permuted) {
    if (kg == 1) BL_RQ(true, 1); else if (kg == 2) BL_RQ(true, 2); else BL_RQ(true, 4);
  } else {
    if (kg == 1) BL_RQ(false, 1); else if (kg == 2) BL_RQ(false, 2); else BL_RQ(false, 4);
  }
#undef BL_RQ
  return cudaGetLastError();
}

}  // namespace bl
