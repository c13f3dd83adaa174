// bl_noalloc.cu - bitlinear_forward_noalloc: the forward with library-owned scratch.
//
// Some callers cannot hand this library a device workspace. A plugin hosted
// by a framework that owns every device byte through its own allocator may
// not call cudaMalloc behind that allocator's back. A C program that embeds
// the library may have no device allocator at all. A latency-critical loop may
// not tolerate cudaMalloc, which can synchronise the device. For them this
// entry point takes only inputs and outputs and uses a fixed scratch array
// that lives in the library's device image. It calls no cudaMalloc, cudaFree
// or other allocating routine.
#include "bitlinear.h"
#include "bl_internal.h"

#include <mutex>

namespace {

// The scratch: one copy per GPU that loads this library, held until the
// process exits. It is laid out like the workspace of bitlinear_forward; its
// first word is the device error word of the calls that use it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[BITLINEAR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

std::mutex g_lookup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// symbol's name is only a host-side stand-in, never a device address, so the
// address is looked up with that device current and cached. Only a successful
// lookup is cached: after a failure (for example a first call made during
// stream capture) the runtime's error is cleared and the next call tries again.
void* scratch_on_current_device(int* status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = BL_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_lookup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      *status = BL_ERR_CUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  *status = BL_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int bitlinear_forward_noalloc(const float* x, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                         const float* D, float* y, bl_stream_t stream) {
  // Reject work that does not fit the fixed scratch before touching the GPU.
  if (M < 0 || K < 0 || N < 0) return BL_ERR_SHAPE;
  if (bitlinear_workspace_size(M, N, K) > (size_t)BITLINEAR_NOALLOC_SCRATCH_BYTES) return BL_ERR_WORKSPACE;
  if (M == 0 || N == 0) return bitlinear_forward(x, M, N, K, packed, D, y, nullptr, 0, stream);
  int st = BL_OK;
  void* scratch = scratch_on_current_device(&st);
  if (st != BL_OK) return st;
  // Nothing in the scratch needs to start at zero: the first kernel of the
  // forward clears the error word, and the quantised activations, scales
  // and row sums are written in full before they are read.
  return bitlinear_forward(x, M, N, K, packed, D, y, scratch, (size_t)BITLINEAR_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int bitlinear_noalloc_error(bl_stream_t stream) {
  int st = BL_OK;
  void* scratch = scratch_on_current_device(&st);
  if (st != BL_OK) return st;
  return bitlinear_workspace_error(scratch, (size_t)BITLINEAR_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int bitlinear_noalloc_selftest_wait_timeout(uint64_t limit_ns, bl_stream_t stream) {
  int st = BL_OK;
  void* scratch = scratch_on_current_device(&st);
  if (st != BL_OK) return st;
  return bitlinear_selftest_wait_timeout(scratch, (size_t)BITLINEAR_NOALLOC_SCRATCH_BYTES, limit_ns, stream);
}
