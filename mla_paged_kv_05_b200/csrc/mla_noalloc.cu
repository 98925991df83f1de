// mla_decode_noalloc: one decode step (plan + run) whose scratch workspace is a
// fixed array compiled into this library instead of memory the caller provides.
//
// Who needs this: a caller that cannot hand the library a device buffer of its
// own - for example code that reaches the library through a foreign-function
// layer with no CUDA allocator binding, a process whose device memory is owned
// by a pool it cannot carve from, or a latency-critical loop that is not
// allowed to allocate (allocation can block, fragment, or be illegal in the
// state the caller is in). Such a caller still passes its own inputs and
// outputs; only the workspace comes from here.
//
// Costs and limits:
//   * every GPU that loads this library holds kNoAllocScratchBytes of device
//     memory for the scratch array until the process exits;
//   * shapes whose workspace would exceed that size are rejected;
//   * all calls share the one array: two calls whose work overlaps on the GPU
//     (different streams, or host threads racing) corrupt each other's results.
//     Calls must be ordered, e.g. issued on one stream.
//   * the first call on a device looks up the array's device address, and so
//     does the first call after that device's context changed (a
//     cudaDeviceReset reloads the library's device code); make those calls
//     before any stream capture begins.
// Nothing in the array must start at zero: the planner rewrites the plan and
// clears the flag word on every call, and partial results are written before
// they are read.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla_decode.h"
#include "mla_common.cuh"
#include "mla_launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = MLA_NOALLOC_SCRATCH_BYTES;

// The scratch array. Host code must not use this name as a device address: on
// the host it only stands in for the symbol; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
struct ScratchAddr {
  CUcontext ctx = nullptr;   // the context the address was looked up in
  void* ptr = nullptr;
};
ScratchAddr g_noalloc_addr[64];

// The current context of the calling thread (nullptr if the lookup fails).
CUcontext current_context() {
  using GetCtx = CUresult (*)(CUcontext*);
  static GetCtx fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCtx>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Once per device and context, with that device current: the device address of
// the array. A device reset (or a primary context torn down and created again)
// loads the module anew, so the address is looked up again when the current
// context is not the one it was found in.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const CUcontext ctx = current_context();   // nullptr before the runtime has bound one to this thread
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  ScratchAddr& a = g_noalloc_addr[dev];
  if (a.ptr == nullptr || ctx == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    a.ptr = p;
    a.ctx = current_context();
  }
  *out = a.ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" MLA_API int mla_decode_noalloc(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                                          const int32_t* block_table, const int32_t* seqlens, void* out,
                                          float* lse, int batch, int max_pages_per_seq, int q_len, int heads,
                                          float scale, void* stream) {
  // Workspace this shape needs (host-side size query; validates the shape).
  size_t need = 0;
  int st = mla_decode_plan(nullptr, nullptr, 0, batch, max_pages_per_seq, q_len, heads, kv_dtype, 0, nullptr, &need,
                           nullptr, stream);
  if (st != MLA_OK) return st;
  if (need > kNoAllocScratchBytes)
    return mla::set_last_error(MLA_ERR_WORKSPACE_TOO_SMALL,
                               "mla_decode_noalloc: this shape needs %zu bytes of workspace, more than the %zu "
                               "bytes of built-in scratch (MLA_NOALLOC_SCRATCH_BYTES); use mla_decode_plan/run "
                               "with a caller-owned workspace",
                               need, kNoAllocScratchBytes);
  void* ws = nullptr;
  const cudaError_t e = noalloc_scratch(&ws);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return mla::set_last_error(MLA_ERR_CUDA, "mla_decode_noalloc: cudaGetSymbolAddress(scratch): %s",
                               cudaGetErrorString(e));
  }
  size_t cap = kNoAllocScratchBytes;
  st = mla_decode_plan(seqlens, block_table, num_pages, batch, max_pages_per_seq, q_len, heads, kv_dtype, 0, ws, &cap,
                       nullptr, stream);
  if (st != MLA_OK) return st;
  return mla_decode_run(q, kv_cache, num_pages, kv_dtype, block_table, seqlens, out, lse, batch, max_pages_per_seq,
                        q_len, heads, scale, ws, kNoAllocScratchBytes, stream);
}
