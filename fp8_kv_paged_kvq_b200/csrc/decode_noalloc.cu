// kvq_decode_noalloc: FP8 decode whose scratch lives in a fixed device array
// owned by the library, for callers that cannot allocate device memory.
//
// Who needs it: some hosts of this library own every byte of device memory
// themselves and forbid plug-ins from allocating (an inference engine that
// hands out only pre-reserved pools), and some serving loops run under a
// rule that no allocation may happen after start-up (allocation can
// synchronize the device or fail under fragmentation in the middle of a
// decode step).  Such callers can still pass inputs and outputs, but cannot
// provide the split-KV workspace that kvq_decode asks for.
//
// The array below is that workspace.  Its size is fixed at build time, so
// every GPU that loads libkvq holds it for the life of the process, and all
// calls on a device share it: two calls that overlap on the GPU (for
// example on two streams without an ordering between them) race on it.
// Nothing in it has to start at zero: the decode kernel writes every entry
// it later reads (the unit prefix and each partial result) within the same
// call, so the contents left by the previous call are never used.
#include <mutex>

#include "kvq.h"
#include "kvq_decode.h"

namespace kvq {
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t{8} << 20;   // 8 MiB per device

static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;

// Device address of g_static_workspace on the current device.  The first
// call on a device looks it up with cudaGetSymbolAddress (with that device
// current) and caches it; later calls only read the cache.
void* static_workspace_on_current_device() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace kvq

extern "C" kvq_status kvq_decode_noalloc(const kvq_cache* cache, const void* q,
                                         int32_t num_q_heads, const int32_t* block_table,
                                         int32_t max_pages, const int32_t* seq_lens, int32_t B,
                                         const uint8_t* abort_mask, float sm_scale, float* out,
                                         float* lse, int32_t num_ctas, void* stream) {
  void* ws = kvq::static_workspace_on_current_device();
  if (ws == nullptr) return KVQ_ERR_CUDA;
  // Same checks and launches as kvq_decode; a batch whose workspace would not
  // fit in the fixed array is rejected with KVQ_ERR_WORKSPACE before any work
  // is enqueued.
  return kvq::decode_common(true, cache, q, num_q_heads, block_table, max_pages, seq_lens, B,
                            abort_mask, sm_scale, out, lse, ws, kvq::kStaticWorkspaceBytes,
                            num_ctas, stream);
}
