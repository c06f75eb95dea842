// kq_linear_noalloc: the whole layer with the activation workspace taken from a
// fixed-size array that lives in this library's device image, so the caller passes no
// workspace and nothing is allocated.
//
// The array is a file-scope __device__ object: it comes into existence when the module
// is loaded on a device and is never freed or resized. Its address on the current
// device is looked up once (cudaGetSymbolAddress, under a lock) by the first call made
// with that device current and cached per device id. After that a call only checks the
// size, clears the error word at the head of the array (kq_quantize_act does this as
// its first enqueued operation) and enqueues the same kernels kq_linear does; every
// other byte the GEMM reads (codes, scales with their padding, means, U) is rewritten
// by the quantize step of the same call, so stale contents of an earlier call never
// reach the output.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/kq.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_workspace[KQ_NOALLOC_WORKSPACE_BYTES];

// Per-device address of g_noalloc_workspace, filled on first use of each device.
kq_status workspace_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KQ_ERR_CUDA;
  static std::mutex mu;
  static std::vector<void*> addr;
  std::lock_guard<std::mutex> g(mu);
  if (static_cast<int>(addr.size()) <= dev) addr.resize(dev + 1, nullptr);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr)
      return KQ_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return KQ_OK;
}

}  // namespace

extern "C" kq_status kq_linear_noalloc(const kq_layer_desc* desc, const void* weights,
                                        const void* X_bf16, int32_t M, void* Y, int32_t out_dtype,
                                        kq_stream_t stream) {
  const size_t need = kq_act_bytes(desc, M);
  // an invalid descriptor or M gives 0: let kq_linear report which argument is wrong
  // (it returns before touching the device when the workspace pointer is null)
  if (need == 0) return kq_linear(desc, weights, X_bf16, M, Y, out_dtype, nullptr, 0, stream);
  if (need > KQ_NOALLOC_WORKSPACE_BYTES) return KQ_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  const kq_status s = workspace_for_current_device(&ws);
  if (s != KQ_OK) return s;
  return kq_linear(desc, weights, X_bf16, M, Y, out_dtype, ws, KQ_NOALLOC_WORKSPACE_BYTES, stream);
}
