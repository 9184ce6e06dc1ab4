// noalloc.cu -- forward attention for callers that cannot allocate device memory.
//
// Some callers are handed only their input and output buffers. One example is a
// plugin inside a host framework that owns every device allocation and gives the
// plugin no allocator. Another is a latency-critical loop that must not call
// cudaMalloc after start-up, because cudaMalloc can synchronise the device. For
// them, entmax_attn_fwd_noalloc runs the same forward kernel as entmax_attn_fwd,
// but the scratch memory (status word, block masks, per-tile counters, sum g,
// Ot) comes from a fixed array in this file instead of a caller-provided workspace.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/entmax_attn.h"
#include "kernels.h"

namespace entmax {
size_t fwd_workspace_bytes(const entmax_attn_desc* d);   // abi.cu: the forward's part of the workspace
}

namespace {

constexpr int kMaxDevices = 64;

// The scratch itself: one copy per GPU that loads the library, held until exit.
__device__ __align__(256) unsigned char g_scratch[ENTMAX_NOALLOC_SCRATCH_BYTES];

// Device address of g_scratch, per device. The host-side symbol g_scratch is only a
// stand-in for the device array; a kernel must be given this address instead.
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_setup_mutex;

// First call on a device: look up the device address of the scratch array, with
// that device current. Returns nullptr on failure.
void* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  p = g_scratch_addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

namespace entmax {
void* noalloc_scratch() { return scratch_for_current_device(); }
}  // namespace entmax

extern "C" entmax_status entmax_attn_fwd_noalloc(const entmax_attn_desc* desc, const void* Q, const void* K,
                                                 const void* V, float* O, float* tau, void* stream) {
  // Only the forward's part of the workspace is needed (status, masks, counters, sum g,
  // Ot and the fp16 copy of V); the backward-only parts come after it in the layout.
  const size_t need = entmax::fwd_workspace_bytes(desc);
  if (need == 0) return ENTMAX_EINVAL;
  if (need > (size_t)ENTMAX_NOALLOC_SCRATCH_BYTES) return ENTMAX_EUNSUPPORTED;   // problem too large
  void* scratch = scratch_for_current_device();
  if (!scratch) return ENTMAX_ECUDA;
  // entmax_attn_fwd clears the status word and the transposed mask (the parts that
  // must start at zero) on `stream` before its kernel runs.
  return entmax_attn_fwd(desc, Q, K, V, O, tau, scratch, stream);
}
