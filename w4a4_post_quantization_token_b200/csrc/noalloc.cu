// kq_linear_noalloc: the whole layer with the activation workspace taken from a
// fixed-size array that lives in this library's device image, so the caller passes no
// workspace and nothing is allocated.
//
// The array is a file-scope __device__ object: it comes into existence when the module
// is loaded in a device context and is never freed or resized. In host code its name is
// only a stand-in, so its device address is looked up (cudaGetSymbolAddress, under a
// lock) by the first call made in a given context and cached per device together with
// that context's unique id. A later call whose current context has another id (the
// primary context was reset and the module loaded again, possibly at another address)
// looks the address up again instead of reusing a stale one. After that a call only
// checks the size, clears the error word at the head of the array (kq_quantize_act does
// this as its first enqueued operation) and enqueues the same kernels kq_linear does;
// every other byte the GEMM reads (codes, scales with their padding, means, U) is
// rewritten by the quantize step of the same call, so stale contents of an earlier call
// never reach the output.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/kq.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_workspace[KQ_NOALLOC_WORKSPACE_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 when none is current or the driver
// cannot say). Driver entry points are looked up once; no driver library is linked.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  CUcontext ctx = nullptr;
  if (get_current == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id != nullptr && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(ctx));
}

// Address of g_noalloc_workspace in the current device's current context.
kq_status workspace_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KQ_ERR_CUDA;
  struct Entry { void* addr = nullptr; unsigned long long ctx = 0; };
  static std::mutex mu;
  static std::vector<Entry> cache;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> g(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  Entry& e = cache[dev];
  if (e.addr == nullptr || ctx == 0 || e.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr)
      return KQ_ERR_CUDA;
    e.addr = p;
    e.ctx = current_context_id();        // the look-up made the context current if none was
  }
  *out = e.addr;
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
