// bl_device.cuh - device helpers shared by the libbitlinear kernels:
// constants of the numeric definition, workspace layout, mbarrier waits with a
// time limit, TMA loads and tcgen05 (TMEM / UMMA) wrappers for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bl {

// ---------------------------------------------------------------- numerics
// Floor applied to mean(|W|) and to max|x| (an all-zero tensor or token).
constexpr float kFloor = 1e-5f;
constexpr float kQmax = 127.0f;
constexpr int64_t kMaxK = 131072;

// ----------------------------------------------------------- workspace ---
// Forward workspace: [header 256 B | s_x fp32[M] | rowsum int32[M] | q int8[M*K]]
// The header's first word is the device error word.
constexpr size_t kHeaderBytes = 256;
__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
__host__ __device__ inline size_t ws_sx_off(int64_t M) { (void)M; return kHeaderBytes; }
__host__ __device__ inline size_t ws_rowsum_off(int64_t M) { return kHeaderBytes + align256(4 * (size_t)M); }
__host__ __device__ inline size_t ws_q_off(int64_t M) { return ws_rowsum_off(M) + align256(4 * (size_t)M); }
__host__ __device__ inline size_t ws_forward_bytes(int64_t M, int64_t K) {
  return ws_q_off(M) + align256((size_t)M * (size_t)K);
}

// Device error codes written into the error word (first failure wins).
enum DevErr : uint32_t {
  kDevOk = 0,
  kDevTimeoutProducer = 0x101,
  kDevTimeoutMma = 0x102,
  kDevTimeoutUnpack = 0x103,
  kDevTimeoutEpilogue = 0x104,
  kDevTimeoutDrain = 0x105,
  kDevTimeoutSelftest = 0x1FF,
};

// ------------------------------------------------------------- general ---
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------ mbarrier ---
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`. Gives up when another role has aborted
// (shared flag) or after `limit_ns`; on its own timeout it raises the abort
// flag and records `code` in the device error word. Returns true on success.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any healthy wait

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* err_word, uint32_t code,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        if (abort_flag != nullptr) *abort_flag = 1;
        if (err_word != nullptr) atomicCAS(err_word, 0u, code);
        return false;
      }
    }
  }
}

// As mbar_try_wait, but a thread whose phase is not complete is suspended
// until it completes or `suspend_ns` elapses, instead of returning at once:
// waiting warps then take no issue slots from the warps that compute.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// mbar_wait with suspended waiting (the abort flag and the time limit are
// checked each time the suspension ends).
constexpr uint32_t kSuspendNs = 50000;  // 50 us: a waiting warp wakes at the phase or after this

__device__ __forceinline__ bool mbar_wait_suspend(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint32_t* err_word, uint32_t code,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_suspend(bar, parity, kSuspendNs)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (abort_flag != nullptr) *abort_flag = 1;
      if (err_word != nullptr) atomicCAS(err_word, 0u, code);
      return false;
    }
  }
}

// ----------------------------------------------------------------- TMA ---
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, int32_t c0, int32_t c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled store of one box from shared memory (bulk-group completion).
// Elements outside the tensor's bounds are not written.
__device__ __forceinline__ void tma_store_2d(const void* tmap, int32_t c0, int32_t c1, const void* smem_src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1), "r"(smem_u32(smem_src))
               : "memory");
}
// As tma_store_2d, but each element is added to the one in global memory
// (fp32: one IEEE round-to-nearest addition per element).
__device__ __forceinline__ void tma_reduce_add_2d(const void* tmap, int32_t c0, int32_t c1, const void* smem_src) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1), "r"(smem_u32(smem_src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of all committed bulk stores have been read.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most one committed bulk-store group still reads its source.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until all committed bulk stores have completed.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- tcgen05 ---
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::i8, int32 accumulate.
__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor: s32 accumulator, signed 8-bit A and B, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_i8(int M, int N) {
  return (2u << 4)                        // c_format = S32
         | (1u << 7)                      // a_format = signed int8
         | (1u << 10)                     // b_format = signed int8
         | (uint32_t(N >> 3) << 17)       // n_dim
         | (uint32_t(M >> 4) << 24);      // m_dim
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the layout a SWIZZLE_128B TMA box of 128-byte rows writes).
__device__ __forceinline__ uint64_t umma_sdesc_sw128(const void* smem) {
  const uint64_t addr = smem_u32(smem);
  return ((addr & 0x3FFFFull) >> 4)   // start address
         | (1ull << 16)               // leading byte offset (unused with swizzle)
         | (64ull << 32)              // stride byte offset = 1024 B
         | (1ull << 46)               // descriptor version (sm_100)
         | (2ull << 61);              // layout: SWIZZLE_128B
}

// 32 lanes x 32 bit, 32 consecutive columns per thread.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------ epilogue ---
// y = RN(RN(float(acc) / s_x) * d), the two-step rescale of the definition.
// float(acc) is exact for |acc| <= 2^24 (the library's K <= 131072 keeps every
// accumulator within that) and the IEEE division __fdiv_rn is correctly
// rounded, so both steps are the single fp32 roundings the definition names.
__device__ __forceinline__ float rescale(int32_t acc, float s_x, float d) {
  return __fmul_rn(__fdiv_rn(__int2float_rn(acc), s_x), d);
}

// RN(a / s) for an integer-valued a (|a| <= 2^24) and s > 0, given r = RN(1/s)
// (one division per token instead of one per output). Markstein's correction
// (IBM J. Res. Dev. 34(1), 1990; Muller et al., "Handbook of Floating-Point
// Arithmetic", division with a fused multiply-add): if r is within half an
// ulp of 1/s and q within one ulp of a/s, the residual e = a - s*q is exact in
// one FMA and RN(q + e*r) is the correctly rounded quotient. q0 = RN(a*r) may
// be up to ~1.5 ulp off, so a first correction brings it within one ulp and
// the second yields RN(a/s). A quotient at the edge of the fp32 range (only
// for max|x| beyond ~1e33) takes the IEEE division instead.
__device__ __forceinline__ float div_rn_by_rcp(float a, float s, float r) {
  float q = __fmul_rn(a, r);
  float e = __fmaf_rn(-q, s, a);
  q = __fmaf_rn(e, r, q);
  e = __fmaf_rn(-q, s, a);
  q = __fmaf_rn(e, r, q);
  if (!(fabsf(q) < 0x1p127f)) q = __fdiv_rn(a, s);
  return q;
}

// The rescale y = RN(RN(float(acc) / s_x) * d) with r = RN(1 / s_x) given.
__device__ __forceinline__ float rescale_rcp(int32_t acc, float s_x, float r, float d) {
  return __fmul_rn(div_rn_by_rcp(__int2float_rn(acc), s_x, r), d);
}

// Inputs are fp32, or bf16 given as 16-bit patterns. A bf16 is the upper half
// of the fp32 with the same value, so widening it is exact. load4 reads the
// four consecutive elements 4*i4 .. 4*i4+3 (16 bytes of fp32 or 8 of bf16).
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

template <bool kBf16>
__device__ __forceinline__ float4 load4(const void* p, int64_t i4) {
  if (kBf16) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i4);
    return make_float4(bf16_bits_to_float(v.x & 0xFFFFu), bf16_bits_to_float(v.x >> 16),
                       bf16_bits_to_float(v.y & 0xFFFFu), bf16_bits_to_float(v.y >> 16));
  }
  return __ldg(reinterpret_cast<const float4*>(p) + i4);
}

// As load4, with ordinary (coherent) loads, for data that the grid this
// launch depends on may have written: a read-only-path load counts as
// invariant memory, so the compiler may hoist it above griddepcontrol.wait.
template <bool kBf16>
__device__ __forceinline__ float4 load4_dep(const void* p, int64_t i4) {
  if (kBf16) {
    const uint2 v = reinterpret_cast<const uint2*>(p)[i4];
    return make_float4(bf16_bits_to_float(v.x & 0xFFFFu), bf16_bits_to_float(v.x >> 16),
                       bf16_bits_to_float(v.y & 0xFFFFu), bf16_bits_to_float(v.y >> 16));
  }
  return reinterpret_cast<const float4*>(p)[i4];
}

// Ternary code of one weight: clamp(rint(RN(w*s)), -1, 1) + 1, in {0, 1, 2}.
__device__ __forceinline__ uint32_t code_plus_one(float w, float s) {
  int c = __float2int_rn(__fmul_rn(w, s));
  c = c < -1 ? -1 : (c > 1 ? 1 : c);
  return static_cast<uint32_t>(c + 1);
}

// int8 activation code: clamp(rint(RN(x*s_x)), -128, 127).
__device__ __forceinline__ int quant_i8(float x, float s_x) {
  int v = __float2int_rn(__fmul_rn(x, s_x));
  return v < -128 ? -128 : (v > 127 ? 127 : v);
}

// int8 activation code clamp(rint(RN(x * s_x)), -128, 127) for a token scale
// s_x = RN(127 / max(max|x|, floor)) and |x| <= max|x|: then |RN(x * s_x)| is at
// most 127 * (1 + 2^-23), far below 2^22. In that range adding 1.5 * 2^23
// rounds to an integer with the fp32 rounding (half to even) and leaves it in
// the low significand bits: the same value as the conversion instruction,
// with one FADD and one integer subtract instead.
__device__ __forceinline__ int quant_code(float x, float s_x) {
  const int v = __float_as_int(__fadd_rn(__fmul_rn(x, s_x), 12582912.0f)) - 0x4B400000;
  return v < -128 ? -128 : (v > 127 ? 127 : v);
}

// ------------------------------------------------------- exact mean square
// Bins of the exact sum of squares of fp32 values, used by the RMSNorm
// quantisers when the fp64 sum cannot decide the fp32 rounding of mean(x^2):
constexpr int kRmsBins = 544;  // x^2 = m^2 * 2^(2(ee-1)) units of 2^-298; m^2 split in 24-bit halves

// Correctly rounded fp32 of (sum_b bins[b] * 2^b) / K * 2^-298, by long
// division on 32-bit limbs (one thread). bins[b] < 2^41.
static __device__ __noinline__ float mean_square_exact_f32(const unsigned long long* bins, uint32_t K) {
  constexpr int L = 19;  // 608 bits: bins below 2^41 at shifts < 544
  uint32_t S[L];
  for (int i = 0; i < L; ++i) S[i] = 0u;
  for (int b = 0; b < kRmsBins; ++b) {
    const unsigned long long v = bins[b];
    if (v == 0ull) continue;
    const int limb = b >> 5, bit = b & 31;
    uint32_t parts[3];
    parts[0] = (uint32_t)(v << bit);
    parts[1] = bit == 0 ? (uint32_t)(v >> 32) : (uint32_t)(v >> (32 - bit));
    parts[2] = bit == 0 ? 0u : (uint32_t)((v >> 32) >> (32 - bit));
    unsigned long long carry = 0ull;
    for (int i = limb; i < L; ++i) {
      const unsigned long long add = (i - limb < 3 ? parts[i - limb] : 0u);
      const unsigned long long t = (unsigned long long)S[i] + add + carry;
      S[i] = (uint32_t)t;
      carry = t >> 32;
      if (i - limb >= 2 && carry == 0ull) break;
    }
  }
  // Q = floor(S / K), remainder r (K < 2^18, so r * 2^32 + limb fits 64 bits).
  uint32_t Q[L];
  unsigned long long r = 0ull;
  for (int i = L - 1; i >= 0; --i) {
    const unsigned long long cur = (r << 32) | S[i];
    Q[i] = (uint32_t)(cur / K);
    r = cur % K;
  }
  int lead = -1;
  for (int i = L - 1; i >= 0 && lead < 0; --i)
    if (Q[i]) lead = 32 * i + 31 - __clz(Q[i]);
  if (lead < 0) return 0.0f;  // below 2^-298: rounds to zero
  auto qbit = [&](int i) -> uint32_t { return (Q[i >> 5] >> (i & 31)) & 1u; };
  const int E = lead - 298;                    // value = 1.xxx * 2^E
  const int qe = E - 23 > -149 ? E - 23 : -149;  // exponent of the last significand bit
  const int p = qe + 298;                      // its bit position in Q (>= 149)
  uint32_t sig = 0u;
  for (int i = lead; i >= p; --i) sig = (sig << 1) | qbit(i);
  const uint32_t round_bit = qbit(p - 1);
  uint32_t sticky = r != 0ull ? 1u : 0u;
  for (int i = p - 2; i >= 0 && !sticky; --i) sticky |= qbit(i);
  if (round_bit && (sticky || (sig & 1u))) ++sig;
  // sig * 2^qe: subnormal when qe == -149 and sig < 2^23; a carry to 2^24 moves up one binade.
  if (qe == -149 && sig < (1u << 23)) return __uint_as_float(sig);
  int e2 = qe + 23;
  if (sig == (1u << 24)) {
    sig >>= 1;
    ++e2;
  }
  return __uint_as_float(((uint32_t)(e2 + 127) << 23) | (sig & 0x7FFFFFu));
}

// Adds x^2 to the bins, exactly: |x| = m * 2^(ee-1) units of 2^-149 (ee the
// biased exponent, at least 1), so x^2 = m^2 * 2^(2(ee-1)) units of 2^-298,
// and m^2 < 2^48 goes in as two 24-bit halves.
__device__ __forceinline__ void rms_bins_add(unsigned long long* bins, float x) {
  const uint32_t b = __float_as_uint(x) & 0x7FFFFFFFu;
  const uint32_t e = b >> 23;
  const unsigned long long mm = (b & 0x7FFFFFu) | (e != 0 ? 0x800000u : 0u);
  if (mm == 0ull) return;
  const int sh = 2 * ((int)(e > 1 ? e : 1) - 1);
  const unsigned long long sq = mm * mm;
  atomicAdd(&bins[sh], sq & 0xFFFFFFull);
  atomicAdd(&bins[sh + 24], sq >> 24);
}

// The 4x4 byte transpose used for the kernel-private activation order: inside
// every group of 16 columns, position 4*c + b holds column 4*b + c. This is
// the order in which `(word >> 2c) & 0x03030303` presents the codes of a
// packed word, so unpacking needs no byte shuffles.
__host__ __device__ constexpr int perm16(int p) { return 4 * (p & 3) + ((p >> 2) & 3); }

}  // namespace bl
