// bl_internal.h - declarations shared by the libbitlinear translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bl_device.cuh"

#include <cudaTypedefs.h>

namespace bl {

// Pack workspace: header (the sticky status word at 0, this call's status at
// 4, a count of finished CTAs at 8, mean_c and s at 16/20) + bins:
// kPackBins sums of significands by weight (bin b weighs 2^(max(b,1)-1) units
// of 2^-149) and, at kPackNonFiniteBin, a count of non-finite weights.
constexpr int kPackBins = 320;
constexpr int kPackNonFiniteBin = kPackBins - 1;
// After the bins: one fp64 partial sum of |W| per CTA of the first pass.
constexpr int kPackSumBlocks = 1024;
constexpr size_t kPackWsBytes = kHeaderBytes + kPackBins * sizeof(unsigned long long) + kPackSumBlocks * sizeof(double);

// Decode path (bl_decode.cu): at most 16 tokens per BitLinear, up to 8
// BitLinears per launch; their activation codes and a ring of at least two
// 16-row weight tiles must fit in shared memory.
constexpr int64_t kDecodeMaxM = 16;
constexpr int kDecodeMaxGroup = 8;                     // BitLinears per grouped launch
constexpr int kDecodeSlots = 16;                       // weight tiles tracked per CTA
constexpr int64_t kDecodeSmemShared = 110 * 1024;   // two CTAs per SM (room for the next launch)
constexpr int64_t kDecodeSmemMax = 225 * 1024;      // one CTA per SM

// I2_S conversion (bl_i2s.cu): to_i2s packs `in` (BitLinear words, D_in)
// into I2_S words at `out`; otherwise unpacks I2_S words at `in` into packed
// words at `out` and D_out. err (a device word, not cleared here) gets bit 0
// OR-ed in for a field holding 3 and bit 1 for a scale that is not finite and
// positive (or rows of D_in that differ).
cudaError_t launch_i2s(bool to_i2s, bool quarters, const void* in, void* out, const float* D_in, float* D_out,
                       int64_t N, int64_t K, uint32_t* err, cudaStream_t stream, int sms);

// One decode BitLinear. x: fp32 [M,K], bf16 bit patterns, or (prepared
// input) int8 codes in the forward workspace's private order with s_x (sx)
// and row sums (rs). y fp32 [M,N], or acc int32 [M,N] when acc is non-null.
struct DecCall {
  const void* x;
  const float* sx;
  const int32_t* rs;
  const uint32_t* packed;
  const float* D;
  float* y;
  int32_t* acc;
  int64_t M, N, K;
};

enum DecInput : int { kDecF32 = 0, kDecBf16 = 1, kDecPrepared = 2, kDecRms = 3 };

// Whether one call of M tokens and K columns (rms: with the RMSNorm input
// mode) fits the decode kernel, and whether a group of calls fits one launch.
bool decode_fits(int64_t M, int64_t K, bool rms);
bool decode_group_fits(const DecCall* calls, int n);
// One launch over n calls (all y or all acc). input: a DecInput; prepared and
// RMSNorm inputs take one call (g: norm weight [K], eps). pdl: launch with
// programmatic stream serialization (the packed weights and D may be read
// before the previous kernel in the stream has finished; activations are read
// after it). err: the workspace error word, cleared by the launch.
cudaError_t launch_decode(const DecCall* calls, int n, int input, const float* g, float eps, uint32_t* err, bool pdl,
                          cudaStream_t stream, int num_sms);

// The driver's cuTensorMapEncodeTiled (looked up once), or nullptr.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// W is fp32, or bf16 bit patterns when bf16 (widened exactly).
// clear_sticky: also zero the workspace's first word, where every call ORs in
// its failure (asynchronous packs leave it for bitlinear_pack_status).
cudaError_t launch_pack(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                        bool clear_sticky, cudaStream_t stream, int num_sms);
// err_reset (nullable): the workspace error word, cleared by the kernel.
// x is fp32, or bf16 bit patterns when bf16 (widened exactly).
cudaError_t launch_act_quant(const void* x, bool bf16, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                             bool permuted, cudaStream_t stream, uint32_t* err_reset);
// RMSNorm (weight g [K], eps) then ActQuant, per token; K <= kRmsMaxK.
constexpr int64_t kRmsMaxK = 16384;
cudaError_t launch_rms_act_quant(const float* x, const float* g, float eps, int64_t M, int64_t K, int8_t* q,
                                 float* s_x, int32_t* rowsum, bool permuted, cudaStream_t stream,
                                 uint32_t* err_reset);
// Natural-order int8 codes and scales (bitlinear_quant_act's output) into the
// forward workspace layout (private order, row sums); err_reset as above.
cudaError_t launch_q_prepare(const int8_t* q, const float* s_x, int64_t M, int64_t K, int8_t* wq, float* wsx,
                             int32_t* wrs, cudaStream_t stream, uint32_t* err_reset);
// Expects the permuted activations, s_x and row sums already in the forward
// workspace (launch_act_quant with permuted = true).
cudaError_t launch_gemm(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                        int32_t* acc_out, void* ws, cudaStream_t stream, int num_sms);
// The same tensor-core kernel over the K range [k0, k0 + K) of rows that are
// kfull columns long (k0 % 16 == 0): the weights' words and the workspace's
// activation codes of that range, the row sums of the codes over it (rowsum,
// or the workspace's when null), D[n * dstride], and with accumulate the
// rescaled tile is added to y (one fp32 rounding per element) instead of
// stored.
struct GemmSlice {
  int64_t k0;
  int64_t kfull;
  int dstride;
  bool accumulate;
  const int32_t* rowsum;
};
cudaError_t launch_gemm_slice(int64_t M, int64_t N, int64_t K, const GemmSlice& sl, const uint32_t* packed,
                              const float* D, float* y, int32_t* acc_out, void* ws, cudaStream_t stream,
                              int num_sms);

// Per-256-block scale variant (bl_block.cu): blocks of 256 consecutive
// columns within a row, D fp32 [N, scale_blocks(K)].
constexpr int kScaleBlock = 256;
inline int64_t scale_blocks(int64_t K) { return (K + kScaleBlock - 1) / kScaleBlock; }
constexpr size_t kBlockFwdSmemMax = 200 * 1024;
// status: a device word that gets bit 0 OR-ed in for a block holding a
// non-finite weight (that block's words and scale are left unwritten).
// W is fp32, or bf16 bit patterns when bf16 (widened exactly).
cudaError_t launch_pack_blocks(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D,
                               uint32_t* status, cudaStream_t stream, int num_sms);
// Tokens per CTA tile of the block forward (its activation codes fit in
// kBlockFwdSmemMax of shared memory); always >= 1 for K <= kMaxK.
int block_forward_tile(int64_t M, int64_t K);
// One token with K % 256 == 0 and K <= kBlockDecMaxK: a single launch that
// quantises x in every CTA. Otherwise ActQuant into the forward workspace ws
// (private order), then the contraction as its programmatic dependent.
constexpr int kBlockDecMaxK = 32 * kScaleBlock;
// From this many tokens on, the block forward runs one tensor-core GEMM per
// block; its workspace then also holds the per-block row sums of the codes.
constexpr int64_t kBlockGemmMinM = 128;
inline size_t ws_blocks_bytes(int64_t M, int64_t K) {
  return ws_forward_bytes(M, K) + align256(4 * (size_t)M * (size_t)scale_blocks(K));
}
// x is fp32, or bf16 bit patterns when bf16 (widened exactly).
cudaError_t launch_forward_blocks(const void* x, bool bf16, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                  const float* D, float* y, void* ws, cudaStream_t stream, int num_sms);

cudaError_t launch_selftest_wait(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);

}  // namespace bl
