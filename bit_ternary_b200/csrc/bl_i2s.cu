// bl_i2s.cu - I2_S import/export of packed BitLinear weights.
//
// Format ("BitNet-Embeddings I2_S guide", section "I2_S Ternary Packing"):
// ternary codes stored as code + 1 in 2 bits, 128 values per 32-byte block,
// byte = c0 << 6 | c1 << 4 | c2 << 2 | c3, and the fp32 scale 1/mean(|w|)
// appended after the blocks. The blocks run over the flattened row-major
// [N, K] tensor; a short tail block is padded with the code 0 (stored 1).
// Which four values share a byte is not stated, so both groupings are built:
//   consecutive  byte j of a block holds values 4j .. 4j+3 as c0 .. c3;
//   quarters     byte j of a block holds values j, j+32, j+64, j+96.
//
// The BitLinear pack stores value k of a row in bits 2*(k%16) of word k/16
// (LSB first), rows back to back, so the packed buffer is the flattened tensor
// in 32-bit words of 16 values. A block is 8 of those words, or 8 I2_S words
// (4 bytes each). One lane pair converts one block: each lane moves 16 bytes
// in and 16 bytes out (one 16-byte load and one 16-byte store, coalesced
// across the warp), with four such loads in flight per lane. The grid is one
// wave (4 CTAs of 256 threads per SM, 64 registers a thread). HBM-bound: N*K/4 bytes read and N*K/4
// bytes written.
//
//   consecutive: I2_S byte j holds the same four values as byte j%4 of our
//   word j/4, with the field order reversed (c0 is the MSB pair), so a word
//   converts on its own, in both directions, by reversing the four 2-bit
//   fields inside each byte.
//   quarters: I2_S word t of a block (bytes 4t .. 4t+3) draws on byte t%4 of
//   our words t/4, 2 + t/4, 4 + t/4, 6 + t/4 (one per quarter), so the two
//   lanes of a block swap two words before (export) or after (import) a
//   4x4 byte transpose (rows fed in reverse order, which stands in for the
//   field reversal) and a 4x4 transpose of 2-bit fields; both are their own
//   inverses, so import runs them in the opposite order.
#include "bl_internal.h"

namespace bl {
namespace {

constexpr uint32_t kZeroWord = 0x55555555u;  // 16 fields of the code 0 (stored 1)
constexpr uint32_t kErrField3 = 1u;          // a field held 3, which is no code
constexpr uint32_t kErrScale = 2u;           // no finite positive scale (or D rows differ)

struct I2sArgs {
  const uint32_t* in;  // export: packed words; import: I2_S words (blocks, then the scale)
  uint32_t* out;       // export: I2_S words; import: packed words
  const float* D_in;   // export: D [N]
  float* D_out;        // import: D [N]
  int64_t nwords;      // packed words of the tensor, N*K/16
  int64_t nhalves;     // 2 * blocks (one lane per half block)
  int64_t N;
  uint32_t* err;
};

__device__ __forceinline__ uint32_t reverse_fields_in_bytes(uint32_t x) {
  return ((x & 0x03030303u) << 6) | ((x & 0x0C0C0C0Cu) << 2) | ((x & 0x30303030u) >> 2) | ((x & 0xC0C0C0C0u) >> 6);
}

__device__ __forceinline__ bool has_field3(uint32_t w) { return (w & (w >> 1) & 0x55555555u) != 0u; }

__device__ __forceinline__ bool finite_positive(float v) {
  return v > 0.0f && (__float_as_uint(v) & 0x7F800000u) != 0x7F800000u;
}

// A word as a 4x4 matrix of 2-bit fields, row r = byte r, column c = field c
// (bits 8r + 2c): returns its transpose (field (r, c) moves to bits 8c + 2r).
// Two delta swaps: the off-diagonal 2x2 blocks (distance 12 bits), then the
// off-diagonal fields inside each block (distance 6 bits).
__device__ __forceinline__ uint32_t transpose_fields(uint32_t x) {
  uint32_t t = ((x >> 12) ^ x) & 0x0000F0F0u;
  x ^= t ^ (t << 12);
  t = ((x >> 6) ^ x) & 0x00CC00CCu;
  x ^= t ^ (t << 6);
  return x;
}

// Four words as a 4x4 matrix of bytes (row = word, column = byte): transposed
// in place, so byte p of word i becomes byte i of word p.
__device__ __forceinline__ void transpose_bytes(uint32_t& q0, uint32_t& q1, uint32_t& q2, uint32_t& q3) {
  const uint32_t a = __byte_perm(q0, q1, 0x5140), b = __byte_perm(q0, q1, 0x7362);
  const uint32_t c = __byte_perm(q2, q3, 0x5140), d = __byte_perm(q2, q3, 0x7362);
  q0 = __byte_perm(a, c, 0x5410);
  q1 = __byte_perm(a, c, 0x7632);
  q2 = __byte_perm(b, d, 0x5410);
  q3 = __byte_perm(b, d, 0x7632);
}

constexpr int kUnroll = 4;  // half blocks per lane in flight (16-byte loads issued before any store)

template <bool kExport, bool kQuarters>
__device__ __forceinline__ void load_half(const I2sArgs& a, int64_t i, bool active, uint32_t (&w)[4]) {
  w[0] = w[1] = w[2] = w[3] = kZeroWord;
  if (!active) return;
  const int64_t w0 = 4 * i;
  if (!kExport || w0 + 3 < a.nwords) {
    const uint4 v = *reinterpret_cast<const uint4*>(a.in + w0);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (w0 + q < a.nwords) w[q] = a.in[w0 + q];
  }
}

// Converts the half block held in w (this lane's 16 bytes) and stores it;
// returns whether a field holding 3 was seen. All 32 lanes must call it.
template <bool kExport, bool kQuarters>
__device__ __forceinline__ bool convert_store(const I2sArgs& a, int64_t i, bool active, int h, const uint32_t (&w)[4]) {
  bool bad = false;
  const int64_t w0 = 4 * i;
  if (kExport && active) {
#pragma unroll
    for (int q = 0; q < 4; ++q) bad |= (w0 + q < a.nwords) && has_field3(w[q]);
  }
  uint32_t o[4];
  if (!kQuarters) {
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = reverse_fields_in_bytes(w[q]);
  } else if (kExport) {
    // Lane h needs our words h, 2+h (its own w[h], w[2+h]) and 4+h, 6+h
    // (lane 0) or 1, 3 (lane 1) from its partner: each lane sends the
    // partner's w[1-h], w[3-h].
    const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, h ? w[0] : w[1], 1);
    const uint32_t r1 = __shfl_xor_sync(0xFFFFFFFFu, h ? w[2] : w[3], 1);
    const uint32_t own0 = h ? w[1] : w[0], own1 = h ? w[3] : w[2];
    // Q[i] = our word 2i + h, the quarter i source of this lane's bytes.
    // Output word p takes byte p of each Q[i], and field f of source i goes
    // to byte f at bits 6 - 2i. The byte transpose, fed Q3 .. Q0, puts byte p
    // of Q[i] into byte 3 - i of word p; the field transpose then moves field
    // f of byte 3 - i to bits 8f + 2(3 - i) = 8f + 6 - 2i.
    uint32_t Q0 = h ? r0 : own0, Q1 = h ? r1 : own1, Q2 = h ? own0 : r0, Q3 = h ? own1 : r1;
    transpose_bytes(Q3, Q2, Q1, Q0);
    o[0] = transpose_fields(Q3);
    o[1] = transpose_fields(Q2);
    o[2] = transpose_fields(Q1);
    o[3] = transpose_fields(Q0);
  } else {
    // V[i] = our word 2i + h, built from this lane's I2_S bytes 16h .. 16h+15
    // by the inverse steps: the field transpose puts the c_i fields of I2_S
    // word p, LSB first, into byte 3 - i; the byte transpose then gathers
    // byte 3 - i of the four words into word 3 - i, which is V[i].
    uint32_t T0 = transpose_fields(w[0]), T1 = transpose_fields(w[1]), T2 = transpose_fields(w[2]),
             T3 = transpose_fields(w[3]);
    transpose_bytes(T0, T1, T2, T3);
    const uint32_t V[4] = {T3, T2, T1, T0};
    // Lane 0 stores words 0..3 (its V0, V1 and the partner's V0, V1 as
    // words 1, 3); lane 1 stores words 4..7 (its V2, V3 and the partner's
    // V2, V3 as words 4, 6).
    const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, h ? V[0] : V[2], 1);
    const uint32_t r1 = __shfl_xor_sync(0xFFFFFFFFu, h ? V[1] : V[3], 1);
    const uint32_t own0 = h ? V[2] : V[0], own1 = h ? V[3] : V[1];
    o[0] = h ? r0 : own0;
    o[1] = h ? own0 : r0;
    o[2] = h ? r1 : own1;
    o[3] = h ? own1 : r1;
  }
  if (active) {
    if (kExport) {
      *reinterpret_cast<uint4*>(a.out + w0) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) bad |= (w0 + q < a.nwords) && has_field3(o[q]);
      if (w0 + 3 < a.nwords) {
        *reinterpret_cast<uint4*>(a.out + w0) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (w0 + q < a.nwords) a.out[w0 + q] = o[q];
      }
    }
  }
  return bad;
}

template <bool kExport, bool kQuarters>
__global__ void __launch_bounds__(256, 4) i2s_convert_kernel(I2sArgs a) {
  const int lane = threadIdx.x & 31;
  const int h = lane & 1;  // which half of the block this lane holds
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;

  // The loop is uniform across each warp (warp bases and the stride are
  // multiples of 32, and nhalves is even), so the two lanes of a block are
  // always both active or both inactive and the shuffles see the whole warp.
  // Each pass issues kUnroll loads before converting and storing.
  for (int64_t base = gtid - lane; base < a.nhalves; base += stride * kUnroll) {
    uint32_t w[kUnroll][4];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * stride + lane;
      load_half<kExport, kQuarters>(a, i, i < a.nhalves, w[u]);
    }
    bool bad = false;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * stride + lane;
      bad |= convert_store<kExport, kQuarters>(a, i, i < a.nhalves, h, w[u]);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicOr(a.err, kErrField3);
  }

  // The scale, which follows the blocks.
  if (kExport) {
    const float d0 = a.D_in[0];
    bool bad = false;
    for (int64_t n = gtid; n < a.N; n += stride) bad |= a.D_in[n] != d0;
    if (gtid == 0) {
      const float scale = __fdiv_rn(1.0f, d0);
      bad |= !finite_positive(d0) || !finite_positive(scale);
      a.out[4 * a.nhalves] = __float_as_uint(scale);
    }
    if (bad) atomicOr(a.err, kErrScale);
  } else {
    const float scale = __uint_as_float(a.in[4 * a.nhalves]);
    const float d = __fdiv_rn(1.0f, scale);
    if (!finite_positive(scale) || !finite_positive(d)) {
      if (gtid == 0) atomicOr(a.err, kErrScale);
      return;
    }
    for (int64_t n = gtid; n < a.N; n += stride) a.D_out[n] = d;
  }
}

}  // namespace

cudaError_t launch_i2s(bool to_i2s, bool quarters, const void* in, void* out, const float* D_in, float* D_out,
                       int64_t N, int64_t K, uint32_t* err, cudaStream_t stream, int sms) {
  I2sArgs a;
  a.in = static_cast<const uint32_t*>(in);
  a.out = static_cast<uint32_t*>(out);
  a.D_in = D_in;
  a.D_out = D_out;
  a.nwords = N * (K / 16);
  a.nhalves = 2 * ((N * K + 127) / 128);
  a.N = N;
  a.err = err;
  const int threads = 256;
  const int64_t lanes = (a.nhalves + kUnroll - 1) / kUnroll;
  const int64_t work = lanes > N ? lanes : N;
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sms * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (to_i2s) {
    if (quarters)
      i2s_convert_kernel<true, true><<<(unsigned)blocks, threads, 0, stream>>>(a);
    else
      i2s_convert_kernel<true, false><<<(unsigned)blocks, threads, 0, stream>>>(a);
  } else {
    if (quarters)
      i2s_convert_kernel<false, true><<<(unsigned)blocks, threads, 0, stream>>>(a);
    else
      i2s_convert_kernel<false, false><<<(unsigned)blocks, threads, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace bl
