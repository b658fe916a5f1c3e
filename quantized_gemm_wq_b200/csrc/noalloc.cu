// noalloc.cu -- the built-in workspace of wq_gemm_grouped_noalloc.
//
// wq_gemm_grouped needs a device workspace (prepared activations, per-quad
// sums, parked partial sums and tile counters), which its caller allocates.
// Some callers cannot allocate device memory at the point of the call: a
// serving runtime that reserves all GPU memory for its own pool at start-up,
// code running while a CUDA graph is being captured (an allocation there is
// either illegal or ends up baked into the graph), or a real-time decode loop
// where an allocation may synchronise the device or fail under memory
// pressure.  For them the library keeps one fixed workspace per GPU: the
// array below, kStaticWorkspaceBytes long, zero at module load and held by
// every GPU that loads the library until the process exits.  It is reached
// only through its device address, looked up here once per device; the host
// name of the array is a stand-in that must never be given to a kernel.
#include <atomic>
#include <mutex>

#include "grouped.h"

namespace wq {

constexpr size_t kStaticWorkspaceBytes = size_t(8) << 20;   // 8 MiB

static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

namespace {
std::atomic<void*> g_static_ws_addr[64];
std::mutex g_static_ws_mu;
}  // namespace

size_t static_workspace_bytes() { return kStaticWorkspaceBytes; }

// Device address of the built-in workspace on the current device.  The first
// call on a device looks it up (cudaGetSymbolAddress, with that device
// current); later calls return the cached address.
cudaError_t static_workspace(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* p = g_static_ws_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    p = g_static_ws_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
      e = cudaGetSymbolAddress(&p, g_static_ws);
      if (e != cudaSuccess) return e;
      if (!p) return cudaErrorInvalidSymbol;
      g_static_ws_addr[dev].store(p, std::memory_order_release);
    }
  }
  *addr = p;
  return cudaSuccess;
}

}  // namespace wq
