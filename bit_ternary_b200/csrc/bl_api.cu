// bl_api.cu - the extern "C" entry points of libbitlinear (see include/bitlinear.h).
// Host-side validation and dispatch only; all arithmetic of the path runs in
// the kernels of bl_quant.cu, bl_decode.cu, bl_gemm.cu and bl_i2s.cu.
#include "bitlinear.h"
#include "bl_internal.h"

#include <vector>

#include <mutex>

namespace {

constexpr int kAbiVersion = 1;
// From this many tokens on, a decode forward quantises x once into the
// workspace instead of in every CTA of the decode kernel.
constexpr int64_t kDecodeQuantiseOnceM = 4;

#ifndef BL_BUILD_ID
#define BL_BUILD_ID "unknown"
#endif

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// Number of SMs of the current device (cached per device id).
int num_sms_current(int* out_dev = nullptr) {
  static int cache[64];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < 64; ++i) cache[i] = 0;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (out_dev) *out_dev = dev;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = v;
  }
  return cache[dev];
}

int check_k(int64_t K) {
  if (K <= 0 || K > bl::kMaxK || (K % 16) != 0) return BL_ERR_SHAPE;
  return BL_OK;
}

int check_mn(int64_t M, int64_t N) {
  if (M < 0 || N < 0 || M > 0x7FFFFFFF || N > 0x7FFFFFFF) return BL_ERR_SHAPE;
  return BL_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

// x is fp32 [M, K], or bf16 bit patterns when bf16.
int forward_impl(const void* x, bool bf16, int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D,
                 float* y, int32_t* acc, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (M == 0 || N == 0) return BL_OK;
  if (x == nullptr || packed == nullptr || ws == nullptr || (y == nullptr && acc == nullptr) ||
      (y != nullptr && D == nullptr))
    return BL_ERR_NULL;
  if (!aligned16(x) || !aligned16(packed) || (y && !aligned16(y)) || (acc && !aligned16(acc)) ||
      (D && !aligned16(D)) || !aligned256(ws))
    return BL_ERR_ALIGN;
  if (ws_bytes < bitlinear_workspace_size(M, N, K)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  if (bl::decode_fits(M, K, false)) {
    if (M >= kDecodeQuantiseOnceM && acc == nullptr) {
      // Several tokens: quantise them once into the workspace, then the
      // decode kernel copies the codes (a quarter of x's bytes) into every
      // CTA instead of each CTA reading and quantising all of x. The decode
      // launch depends on the quantiser programmatically: its weights start
      // streaming while the quantiser runs.
      cudaError_t e = bl::launch_act_quant(x, bf16, M, K, reinterpret_cast<int8_t*>(base + bl::ws_q_off(M)),
                                           reinterpret_cast<float*>(base + bl::ws_sx_off(M)),
                                           reinterpret_cast<int32_t*>(base + bl::ws_rowsum_off(M)), true, stream,
                                           err);
      if (e != cudaSuccess) return BL_ERR_CUDA;
      const bl::DecCall call{base + bl::ws_q_off(M), reinterpret_cast<const float*>(base + bl::ws_sx_off(M)),
                             reinterpret_cast<const int32_t*>(base + bl::ws_rowsum_off(M)), packed, D, y, nullptr,
                             M, N, K};
      return cuda_status(bl::launch_decode(&call, 1, bl::kDecPrepared, nullptr, 0.0f, err, true, stream, sms));
    }
    const bl::DecCall call{x, nullptr, nullptr, packed, D, y, acc, M, N, K};
    return cuda_status(
        bl::launch_decode(&call, 1, bf16 ? bl::kDecBf16 : bl::kDecF32, nullptr, 0.0f, err, false, stream, sms));
  }
  cudaError_t e = bl::launch_act_quant(x, bf16, M, K, reinterpret_cast<int8_t*>(base + bl::ws_q_off(M)),
                                       reinterpret_cast<float*>(base + bl::ws_sx_off(M)),
                                       reinterpret_cast<int32_t*>(base + bl::ws_rowsum_off(M)), true, stream, err);
  if (e != cudaSuccess) return BL_ERR_CUDA;
  return cuda_status(bl::launch_gemm(M, N, K, packed, D, y, acc, ws, stream, sms));
}

// Contraction + rescale from prepared activations in the forward workspace
// (private-order codes, s_x, row sums): the decode kernel for M <= 16 when it
// fits, the tensor-core kernel otherwise.
int prepared_contraction(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y, void* ws,
                         cudaStream_t stream, int sms) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (bl::decode_fits(M, K, false)) {
    const bl::DecCall call{base + bl::ws_q_off(M), reinterpret_cast<const float*>(base + bl::ws_sx_off(M)),
                           reinterpret_cast<const int32_t*>(base + bl::ws_rowsum_off(M)), packed, D, y, nullptr,
                           M, N, K};
    return cuda_status(bl::launch_decode(&call, 1, bl::kDecPrepared, nullptr, 0.0f, reinterpret_cast<uint32_t*>(base),
                                         false, stream, sms));
  }
  return cuda_status(bl::launch_gemm(M, N, K, packed, D, y, nullptr, ws, stream, sms));
}

}  // namespace

extern "C" {

int bitlinear_abi_version(void) { return kAbiVersion; }

const char* bitlinear_build_id(void) { return BL_BUILD_ID; }

const char* bitlinear_status_string(int status) {
  switch (status) {
    case BL_OK: return "ok";
    case BL_ERR_NULL: return "null pointer";
    case BL_ERR_SHAPE: return "bad shape (need 0 < K <= 131072, K % 16 == 0, 0 <= M, N < 2^31)";
    case BL_ERR_ALIGN: return "misaligned pointer (device buffers 16 B, workspace 256 B)";
    case BL_ERR_WORKSPACE: return "workspace too small";
    case BL_ERR_NONFINITE: return "weights hold Inf or NaN";
    case BL_ERR_DEVICE: return "device-side failure recorded (bounded wait expired)";
    case BL_ERR_CUDA: return "CUDA runtime error";
    case BL_ERR_UNSUPPORTED: return "device is not sm_100 (B200 class)";
    case BL_ERR_FORMAT: return "I2_S: field holding 3, bad scale, or rows of D that differ";
    default: return "unknown status";
  }
}

int bitlinear_device_check(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BL_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return BL_ERR_CUDA;
  return (major == 10 && minor == 0) ? BL_OK : BL_ERR_UNSUPPORTED;
}

size_t bitlinear_pack_workspace_size(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return bl::kPackWsBytes;
}

static int pack_impl(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                     size_t ws_bytes, bl_stream_t stream, bool sync = true) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (W == nullptr || packed == nullptr || D == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(D) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::kPackWsBytes) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bl::launch_pack(W, bf16, N, K, packed, D, ws, sync, s, sms) != cudaSuccess) return BL_ERR_CUDA;
  if (!sync) return BL_OK;
  uint32_t status = 0;
  if (cudaMemcpyAsync(&status, ws, sizeof(status), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  return status == 0u ? BL_OK : BL_ERR_NONFINITE;
}

static int quant_act_impl(const void* x, bool bf16, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                          bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (M < 0 || M > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (x == nullptr || q == nullptr || s_x == nullptr) return BL_ERR_NULL;
  if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s_x) & 3u) ||
      (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
    return BL_ERR_ALIGN;
  return cuda_status(
      bl::launch_act_quant(x, bf16, M, K, q, s_x, rowsum, false, reinterpret_cast<cudaStream_t>(stream), nullptr));
}

int bitlinear_pack_weights(const float* W, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                           size_t ws_bytes, bl_stream_t stream) {
  return pack_impl(W, false, N, K, packed, D, ws, ws_bytes, stream);
}

int bitlinear_pack_weights_bf16(const uint16_t* W, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                                size_t ws_bytes, bl_stream_t stream) {
  return pack_impl(W, true, N, K, packed, D, ws, ws_bytes, stream);
}

int bitlinear_pack_weights_async(const float* W, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                                 size_t ws_bytes, bl_stream_t stream) {
  return pack_impl(W, false, N, K, packed, D, ws, ws_bytes, stream, false);
}

int bitlinear_pack_status(void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::kPackWsBytes) return BL_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* word = static_cast<uint32_t*>(ws);
  uint32_t status = 0;
  if (cudaMemcpyAsync(&status, word, sizeof(status), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  if (status == 0u) return BL_OK;
  if (cudaMemsetAsync(word, 0, sizeof(status), s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  return BL_ERR_NONFINITE;
}

int bitlinear_quant_act(const float* x, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                        bl_stream_t stream) {
  return quant_act_impl(x, false, M, K, q, s_x, rowsum, stream);
}

int bitlinear_quant_act_bf16(const uint16_t* x, int64_t M, int64_t K, int8_t* q, float* s_x, int32_t* rowsum,
                             bl_stream_t stream) {
  return quant_act_impl(x, true, M, K, q, s_x, rowsum, stream);
}

size_t bitlinear_workspace_size(int64_t M, int64_t N, int64_t K) {
  (void)N;
  if (M < 0 || K < 0) return 0;
  return bl::ws_forward_bytes(M, K);
}

int bitlinear_forward(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D,
                      float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (y == nullptr && M > 0 && N > 0) return BL_ERR_NULL;
  return forward_impl(x, false, M, N, K, packed, D, y, nullptr, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int bitlinear_forward_bf16(const uint16_t* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const float* D, float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (y == nullptr && M > 0 && N > 0) return BL_ERR_NULL;
  return forward_impl(x, true, M, N, K, packed, D, y, nullptr, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int bitlinear_forward_acc(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed, int32_t* acc,
                          void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (acc == nullptr && M > 0 && N > 0) return BL_ERR_NULL;
  return forward_impl(x, false, M, N, K, packed, nullptr, nullptr, acc, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int bitlinear_prepare_act(const float* x, int64_t M, int64_t K, void* ws, size_t ws_bytes, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (M < 0 || M > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (x == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(x) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::ws_forward_bytes(M, K)) return BL_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  return cuda_status(bl::launch_act_quant(x, false, M, K, reinterpret_cast<int8_t*>(base + bl::ws_q_off(M)),
                                          reinterpret_cast<float*>(base + bl::ws_sx_off(M)),
                                          reinterpret_cast<int32_t*>(base + bl::ws_rowsum_off(M)), true,
                                          reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<uint32_t*>(base)));
}

int bitlinear_forward_prepared(int64_t M, int64_t N, int64_t K, const uint32_t* packed, const float* D, float* y,
                               void* ws, size_t ws_bytes, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (M == 0 || N == 0) return BL_OK;
  if (packed == nullptr || D == nullptr || y == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(packed) || !aligned16(D) || !aligned16(y) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::ws_forward_bytes(M, K)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  return prepared_contraction(M, N, K, packed, D, y, ws, reinterpret_cast<cudaStream_t>(stream), sms);
}

int bitlinear_forward_q(const int8_t* q, const float* s_x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                        const float* D, float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (M == 0 || N == 0) return BL_OK;
  if (q == nullptr || s_x == nullptr || packed == nullptr || D == nullptr || y == nullptr || ws == nullptr)
    return BL_ERR_NULL;
  if (!aligned16(q) || !aligned16(packed) || !aligned16(D) || !aligned16(y) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bitlinear_workspace_size(M, N, K)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  st = cuda_status(bl::launch_q_prepare(q, s_x, M, K, reinterpret_cast<int8_t*>(base + bl::ws_q_off(M)),
                                        reinterpret_cast<float*>(base + bl::ws_sx_off(M)),
                                        reinterpret_cast<int32_t*>(base + bl::ws_rowsum_off(M)), s,
                                        reinterpret_cast<uint32_t*>(base)));
  if (st != BL_OK) return st;
  return prepared_contraction(M, N, K, packed, D, y, ws, s, sms);
}

int bitlinear_rmsnorm_quant_act(const float* x, const float* g, float eps, int64_t M, int64_t K, int8_t* q,
                                float* s_x, int32_t* rowsum, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (K > bl::kRmsMaxK || M < 0 || M > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (M == 0) return BL_OK;
  if (x == nullptr || g == nullptr || q == nullptr || s_x == nullptr) return BL_ERR_NULL;
  if (!aligned16(x) || !aligned16(g) || !aligned16(q) || (reinterpret_cast<uintptr_t>(s_x) & 3u) ||
      (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
    return BL_ERR_ALIGN;
  if (!(eps >= 0.0f) || eps > 1e30f) return BL_ERR_SHAPE;
  return cuda_status(bl::launch_rms_act_quant(x, g, eps, M, K, q, s_x, rowsum, false,
                                              reinterpret_cast<cudaStream_t>(stream), nullptr));
}

int bitlinear_forward_rmsnorm(const float* x, const float* g, float eps, int64_t M, int64_t N, int64_t K,
                              const uint32_t* packed, const float* D, float* y, void* ws, size_t ws_bytes,
                              bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (K > bl::kRmsMaxK) return BL_ERR_SHAPE;
  if (M == 0 || N == 0) return BL_OK;
  if (x == nullptr || g == nullptr || packed == nullptr || D == nullptr || y == nullptr || ws == nullptr)
    return BL_ERR_NULL;
  if (!aligned16(x) || !aligned16(g) || !aligned16(packed) || !aligned16(D) || !aligned16(y) || !aligned256(ws))
    return BL_ERR_ALIGN;
  if (!(eps >= 0.0f) || eps > 1e30f) return BL_ERR_SHAPE;
  if (ws_bytes < bitlinear_workspace_size(M, N, K)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (bl::decode_fits(M, K, true)) {
    // Decode sizes: the norm and the quantiser run inside the decode kernel.
    const bl::DecCall call{x, nullptr, nullptr, packed, D, y, nullptr, M, N, K};
    return cuda_status(
        bl::launch_decode(&call, 1, bl::kDecRms, g, eps, reinterpret_cast<uint32_t*>(base), false, s, sms));
  }
  st = cuda_status(bl::launch_rms_act_quant(x, g, eps, M, K, reinterpret_cast<int8_t*>(base + bl::ws_q_off(M)),
                                            reinterpret_cast<float*>(base + bl::ws_sx_off(M)),
                                            reinterpret_cast<int32_t*>(base + bl::ws_rowsum_off(M)), true, s,
                                            reinterpret_cast<uint32_t*>(base)));
  if (st != BL_OK) return st;
  return cuda_status(bl::launch_gemm(M, N, K, packed, D, y, nullptr, ws, s, sms));
}

int64_t bitlinear_block_scales(int64_t K) {
  if (check_k(K) != BL_OK) return 0;
  return bl::scale_blocks(K);
}

static int pack_blocks_impl(const void* W, bool bf16, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                            size_t ws_bytes, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (W == nullptr || packed == nullptr || D == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(D) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::kPackWsBytes) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* word = static_cast<uint32_t*>(ws);
  if (cudaMemsetAsync(word, 0, sizeof(uint32_t), s) != cudaSuccess) return BL_ERR_CUDA;
  if (bl::launch_pack_blocks(W, bf16, N, K, packed, D, word, s, sms) != cudaSuccess) return BL_ERR_CUDA;
  uint32_t status = 0;
  if (cudaMemcpyAsync(&status, word, sizeof(status), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  return status == 0u ? BL_OK : BL_ERR_NONFINITE;
}

size_t bitlinear_blocks_workspace_size(int64_t M, int64_t N, int64_t K) {
  (void)N;
  if (M < 0 || K <= 0 || check_k(K) != BL_OK) return 0;
  return bl::ws_blocks_bytes(M, K);
}

int bitlinear_pack_weights_blocks(const float* W, int64_t N, int64_t K, uint32_t* packed, float* D, void* ws,
                                  size_t ws_bytes, bl_stream_t stream) {
  return pack_blocks_impl(W, false, N, K, packed, D, ws, ws_bytes, stream);
}

int bitlinear_pack_weights_blocks_bf16(const uint16_t* W, int64_t N, int64_t K, uint32_t* packed, float* D,
                                       void* ws, size_t ws_bytes, bl_stream_t stream) {
  return pack_blocks_impl(W, true, N, K, packed, D, ws, ws_bytes, stream);
}

static int forward_blocks_impl(const void* x, bool bf16, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                               const float* D, float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (M == 0 || N == 0) return BL_OK;
  if (x == nullptr || packed == nullptr || D == nullptr || y == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(D) || !aligned16(y) || !aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::ws_blocks_bytes(M, K)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  return cuda_status(
      bl::launch_forward_blocks(x, bf16, M, N, K, packed, D, y, ws, reinterpret_cast<cudaStream_t>(stream), sms));
}

int bitlinear_forward_blocks(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                             const float* D, float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  return forward_blocks_impl(x, false, M, N, K, packed, D, y, ws, ws_bytes, stream);
}

int bitlinear_forward_blocks_bf16(const uint16_t* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                  const float* D, float* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
  return forward_blocks_impl(x, true, M, N, K, packed, D, y, ws, ws_bytes, stream);
}

size_t bitlinear_batch_workspace_size(const bl_linear_call* calls, int count) {
  size_t need = bl::kHeaderBytes;
  if (calls == nullptr || count < 0) return 0;
  for (int i = 0; i < count; ++i) {
    const size_t w = bitlinear_workspace_size(calls[i].M, calls[i].N, calls[i].K);
    need = w > need ? w : need;
  }
  return need;
}

int bitlinear_forward_batch(const bl_linear_call* calls, int count, uint32_t flags, void* ws, size_t ws_bytes,
                            bl_stream_t stream) {
  if (count < 0) return BL_ERR_SHAPE;
  if (count == 0) return BL_OK;
  if (calls == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (flags & ~(uint32_t)(BL_FLAG_STREAM_WEIGHTS_EARLY | BL_FLAG_ONE_LAUNCH_PER_CALL)) return BL_ERR_SHAPE;
  // Validate every call before launching anything.
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    int st = check_k(c.K);
    if (st != BL_OK) return st;
    st = check_mn(c.M, c.N);
    if (st != BL_OK) return st;
    if (c.M == 0 || c.N == 0) continue;
    if (c.x == nullptr || c.packed == nullptr || c.D == nullptr || c.y == nullptr) return BL_ERR_NULL;
    if (!aligned16(c.x) || !aligned16(c.packed) || !aligned16(c.D) || !aligned16(c.y)) return BL_ERR_ALIGN;
  }
  if (ws_bytes < bitlinear_batch_workspace_size(calls, count)) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(ws);
  const bool early = (flags & BL_FLAG_STREAM_WEIGHTS_EARLY) != 0;
  const int max_group = (flags & BL_FLAG_ONE_LAUNCH_PER_CALL) ? 1 : bl::kDecodeMaxGroup;
  // Decode-sized calls are grouped, in order, into launches of up to
  // max_group; every other call runs on its own.
  bl::DecCall group[bl::kDecodeMaxGroup];
  int ng = 0;
  auto flush = [&]() -> int {
    if (ng == 0) return BL_OK;
    const cudaError_t e = bl::launch_decode(group, ng, bl::kDecF32, nullptr, 0.0f, err, early, s, sms);
    ng = 0;
    return cuda_status(e);
  };
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    if (c.M == 0 || c.N == 0) continue;
    const bl::DecCall dc{c.x, nullptr, nullptr, c.packed, c.D, c.y, nullptr, c.M, c.N, c.K};
    if (bl::decode_group_fits(&dc, 1)) {
      if (ng == max_group) {
        const int st = flush();
        if (st != BL_OK) return st;
      }
      group[ng] = dc;
      if (!bl::decode_group_fits(group, ng + 1)) {
        const int st = flush();
        if (st != BL_OK) return st;
        group[0] = dc;
      }
      ++ng;
      continue;
    }
    int st = flush();
    if (st != BL_OK) return st;
    st = forward_impl(c.x, false, c.M, c.N, c.K, c.packed, c.D, c.y, nullptr, ws, ws_bytes, s);
    if (st != BL_OK) return st;
  }
  return flush();
}

// Bytes of x (in) or y (out) that a call stages; calls with no output move nothing.
static size_t staged_bytes(const bl_linear_call& c, bool in) {
  if (c.M <= 0 || c.N <= 0 || c.K < 0) return 0;
  return 4 * (size_t)c.M * (size_t)(in ? c.K : c.N);
}

// Room a staged block takes: its bytes rounded up to 16, so every block starts
// 16-byte aligned.
static size_t staged_room(const bl_linear_call& c, bool in) { return (staged_bytes(c, in) + 15) & ~(size_t)15; }

size_t bitlinear_batch_host_workspace_size(const bl_linear_call* calls, int count) {
  if (calls == nullptr || count < 0) return 0;
  size_t xs = 0, ys = 0;
  for (int i = 0; i < count; ++i) {
    if (calls[i].M < 0 || calls[i].N < 0 || calls[i].K < 0) return 0;
    xs += staged_room(calls[i], true);
    ys += staged_room(calls[i], false);
  }
  return bl::align256(bitlinear_batch_workspace_size(calls, count)) + bl::align256(xs) + bl::align256(ys);
}

int bitlinear_forward_batch_host(const bl_linear_call* calls, int count, uint32_t flags, void* ws, size_t ws_bytes,
                                 bl_stream_t stream) {
  if (count < 0) return BL_ERR_SHAPE;
  if (count == 0) return BL_OK;
  if (calls == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (flags & ~(uint32_t)(BL_FLAG_STREAM_WEIGHTS_EARLY | BL_FLAG_ONE_LAUNCH_PER_CALL)) return BL_ERR_SHAPE;
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    int st = check_k(c.K);
    if (st != BL_OK) return st;
    st = check_mn(c.M, c.N);
    if (st != BL_OK) return st;
    if (c.M == 0 || c.N == 0) continue;
    if (c.x == nullptr || c.packed == nullptr || c.D == nullptr || c.y == nullptr) return BL_ERR_NULL;
    if (!aligned16(c.packed) || !aligned16(c.D)) return BL_ERR_ALIGN;
  }
  if (ws_bytes < bitlinear_batch_host_workspace_size(calls, count)) return BL_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t fw = bl::align256(bitlinear_batch_workspace_size(calls, count));
  size_t xs = 0;
  for (int i = 0; i < count; ++i) xs += staged_room(calls[i], true);
  uint8_t* xdev = base + fw;                    // activations of all calls, back to back
  uint8_t* ydev = base + fw + bl::align256(xs);  // outputs of all calls, back to back
  // Device copies of the calls, pointing into the staging areas.
  std::vector<bl_linear_call> dc(calls, calls + count);
  size_t xo = 0, yo = 0;
  for (int i = 0; i < count; ++i) {
    dc[i].x = reinterpret_cast<const float*>(xdev + xo);
    dc[i].y = reinterpret_cast<float*>(ydev + yo);
    xo += staged_room(calls[i], true);
    yo += staged_room(calls[i], false);
  }
  // Blocks that follow one another both in host memory and in the staging
  // area move in one copy; calls that stage nothing are skipped.
  auto copy_runs = [&](bool in) -> int {
    const char* run_host = nullptr;
    size_t run_off = 0, run_len = 0, off = 0;
    auto flush = [&]() -> int {
      if (run_len == 0) return BL_OK;
      const cudaError_t e =
          in ? cudaMemcpyAsync(xdev + run_off, run_host, run_len, cudaMemcpyHostToDevice, s)
             : cudaMemcpyAsync(const_cast<char*>(run_host), ydev + run_off, run_len, cudaMemcpyDeviceToHost, s);
      run_len = 0;
      return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
    };
    for (int i = 0; i < count; ++i) {
      const size_t b = staged_bytes(calls[i], in);
      if (b == 0) continue;
      const char* h = in ? reinterpret_cast<const char*>(calls[i].x) : reinterpret_cast<const char*>(calls[i].y);
      if (run_len != 0 && (h != run_host + run_len || off != run_off + run_len)) {
        const int st = flush();
        if (st != BL_OK) return st;
      }
      if (run_len == 0) {
        run_host = h;
        run_off = off;
      }
      run_len += b;
      off += staged_room(calls[i], in);
    }
    return flush();
  };
  int st = copy_runs(true);
  if (st != BL_OK) return st;
  st = bitlinear_forward_batch(dc.data(), count, flags, ws, fw, stream);
  if (st != BL_OK) return st;
  return copy_runs(false);
}

size_t bitlinear_host_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return bl::ws_forward_bytes(M, K) + bl::align256(4 * (size_t)M * (size_t)K) +
         bl::align256(4 * (size_t)M * (size_t)N);
}

static int forward_host_impl(const float* x_host, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                             const float* D, float* y_host, void* ws, size_t ws_bytes, bl_stream_t stream,
                             bool sync) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  st = check_mn(M, N);
  if (st != BL_OK) return st;
  if (M == 0 || N == 0) return BL_OK;
  if (x_host == nullptr || y_host == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bitlinear_host_workspace_size(M, N, K)) return BL_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const size_t fw = bl::ws_forward_bytes(M, K);
  float* xd = reinterpret_cast<float*>(base + fw);
  float* yd = reinterpret_cast<float*>(base + fw + bl::align256(4 * (size_t)M * (size_t)K));
  if (cudaMemcpyAsync(xd, x_host, 4 * (size_t)M * (size_t)K, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return BL_ERR_CUDA;
  st = forward_impl(xd, false, M, N, K, packed, D, yd, nullptr, ws, fw, s);
  if (st != BL_OK) return st;
  if (cudaMemcpyAsync(y_host, yd, 4 * (size_t)M * (size_t)N, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BL_ERR_CUDA;
  if (!sync) return BL_OK;
  return cudaStreamSynchronize(s) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

int bitlinear_forward_host(const float* x_host, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const float* D, float* y_host, void* ws, size_t ws_bytes, bl_stream_t stream) {
  return forward_host_impl(x_host, M, N, K, packed, D, y_host, ws, ws_bytes, stream, true);
}

int bitlinear_forward_host_async(const float* x_host, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                 const float* D, float* y_host, void* ws, size_t ws_bytes, bl_stream_t stream) {
  return forward_host_impl(x_host, M, N, K, packed, D, y_host, ws, ws_bytes, stream, false);
}

int bitlinear_workspace_error(void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (ws == nullptr) return BL_ERR_NULL;
  if (ws_bytes < bl::kHeaderBytes) return BL_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  if (word == 0u) return BL_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(word), s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  return BL_ERR_DEVICE;
}

int bitlinear_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, bl_stream_t stream) {
  if (ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::kHeaderBytes) return BL_ERR_WORKSPACE;
  const uint64_t cap = 100000000ull;
  return cuda_status(bl::launch_selftest_wait(static_cast<uint32_t*>(ws), limit_ns < cap ? limit_ns : cap,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

size_t bitlinear_i2s_bytes(int64_t N, int64_t K) {
  if (N < 0 || K < 0) return 0;
  return 32 * (((size_t)N * (size_t)K + 127) / 128) + 4;
}

size_t bitlinear_i2s_workspace_size(void) { return bl::kHeaderBytes; }

// Reads and clears the I2_S status word (after synchronising the stream).
static int i2s_read_status(uint32_t* err, cudaStream_t s) {
  uint32_t status = 0;
  if (cudaMemcpyAsync(&status, err, sizeof(status), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  if (status == 0u) return BL_OK;
  if (cudaMemsetAsync(err, 0, sizeof(status), s) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BL_ERR_CUDA;
  return BL_ERR_FORMAT;
}

// Shared checks of the two I2_S conversions; `sync` clears the status word
// first and reads it back at the end.
static int i2s_impl(bool to_i2s, const void* i2s, const uint32_t* packed, const float* D, int64_t N, int64_t K,
                    int layout, void* ws, size_t ws_bytes, bl_stream_t stream, bool sync) {
  int st = check_k(K);
  if (st != BL_OK) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return BL_ERR_SHAPE;
  if (layout != BL_I2S_CONSECUTIVE && layout != BL_I2S_QUARTERS) return BL_ERR_SHAPE;
  if (i2s == nullptr || packed == nullptr || D == nullptr || ws == nullptr) return BL_ERR_NULL;
  if (!aligned16(i2s) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(D) & 3u) || !aligned256(ws))
    return BL_ERR_ALIGN;
  if (ws_bytes < bl::kHeaderBytes) return BL_ERR_WORKSPACE;
  const int sms = num_sms_current();
  if (sms <= 0) return BL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(ws);
  if (sync && cudaMemsetAsync(err, 0, sizeof(uint32_t), s) != cudaSuccess) return BL_ERR_CUDA;
  const cudaError_t e =
      to_i2s ? bl::launch_i2s(true, layout == BL_I2S_QUARTERS, packed, const_cast<void*>(i2s), D, nullptr, N, K,
                              err, s, sms)
             : bl::launch_i2s(false, layout == BL_I2S_QUARTERS, i2s, const_cast<uint32_t*>(packed), nullptr,
                              const_cast<float*>(D), N, K, err, s, sms);
  if (e != cudaSuccess) return BL_ERR_CUDA;
  return sync ? i2s_read_status(err, s) : BL_OK;
}

int bitlinear_i2s_export(const uint32_t* packed, const float* D, int64_t N, int64_t K, int layout, uint8_t* i2s,
                         void* ws, size_t ws_bytes, bl_stream_t stream) {
  return i2s_impl(true, i2s, packed, D, N, K, layout, ws, ws_bytes, stream, true);
}

int bitlinear_i2s_export_async(const uint32_t* packed, const float* D, int64_t N, int64_t K, int layout,
                               uint8_t* i2s, void* ws, size_t ws_bytes, bl_stream_t stream) {
  return i2s_impl(true, i2s, packed, D, N, K, layout, ws, ws_bytes, stream, false);
}

int bitlinear_i2s_import(const uint8_t* i2s, int64_t N, int64_t K, int layout, uint32_t* packed, float* D, void* ws,
                         size_t ws_bytes, bl_stream_t stream) {
  return i2s_impl(false, i2s, packed, D, N, K, layout, ws, ws_bytes, stream, true);
}

int bitlinear_i2s_import_async(const uint8_t* i2s, int64_t N, int64_t K, int layout, uint32_t* packed, float* D,
                               void* ws, size_t ws_bytes, bl_stream_t stream) {
  return i2s_impl(false, i2s, packed, D, N, K, layout, ws, ws_bytes, stream, false);
}

int bitlinear_i2s_status(void* ws, size_t ws_bytes, bl_stream_t stream) {
  if (ws == nullptr) return BL_ERR_NULL;
  if (!aligned256(ws)) return BL_ERR_ALIGN;
  if (ws_bytes < bl::kHeaderBytes) return BL_ERR_WORKSPACE;
  return i2s_read_status(static_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
