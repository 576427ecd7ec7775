// Decode attention for callers that cannot allocate device memory.
//
// tpa_decode_attention needs a caller-provided workspace for the per-split
// softmax partials whenever it cuts the token range into several splits.
// Some callers have no way to provide one: a plugin running inside an
// inference engine that owns the entire device-memory budget and forbids
// allocations while a request is in flight, or a latency-critical serving
// loop that must never reach cudaMalloc (which can synchronise the whole
// device).  tpa_decode_attention_noalloc serves them from a fixed scratch
// array compiled into the library instead.
//
// The scratch is a file-scope device array of kNoAllocScratchBytes.  Every
// GPU that loads libtpa holds it until the process exits.  Host code only
// sees a host-side stand-in under the array's name, so the device address is
// looked up with cudaGetSymbolAddress, once per device, on the first call
// made with that device current; that first call on each device should
// therefore come before any stream capture (a lookup that fails is not kept,
// and the next call tries again).  All calls on a device share the
// one array, which keeps whatever the previous call left in it: the decode
// kernels write every partial before the merge reads it, so nothing has to
// start at zero, but two calls that overlap on the GPU (different streams,
// no ordering between them) race on the array and corrupt each other's
// results.
#include <mutex>

#include "../../include/tpa.h"
#include "tpa_internal.h"

namespace tpa {

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxNoAllocDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxNoAllocDevices];  // non-null once a lookup on that device has succeeded

// Device address of the scratch array on the current device.  Only a successful lookup is
// kept: a failed one (made during a stream capture, or a transient error) is tried again on
// the next call.
cudaError_t scratch_address(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxNoAllocDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace tpa

extern "C" tpa_status tpa_decode_attention_noalloc(const tpa_cache* cache, const void* q, const int32_t* q_pos,
                                                   float scale, float* out, int32_t max_len, int32_t num_splits,
                                                   int32_t kernel, void* stream) {
  using namespace tpa;
  int32_t splits = num_splits;
  size_t need = tpa_decode_workspace_size(cache, max_len, splits, kernel);
  if (need > kNoAllocScratchBytes) {
    if (num_splits != 0) {
      set_last_error_message(
          "tpa_decode_attention_noalloc: %d splits need %zu bytes of scratch, more than the %zu-byte array "
          "compiled into the library; pass fewer splits (or 0 to let the library pick a count that fits)",
          num_splits, need, kNoAllocScratchBytes);
      return TPA_ERR_WORKSPACE;
    }
    // default plan too large for the array: shrink the split count until the partials fit
    splits = tpa_decode_default_splits(cache, max_len, kernel);
    while (splits > 1 && tpa_decode_workspace_size(cache, max_len, splits, kernel) > kNoAllocScratchBytes)
      splits = splits * 3 / 4 > 0 ? splits * 3 / 4 : 1;
    if (splits < 1) splits = 1;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    set_last_error_message("tpa_decode_attention_noalloc: cudaGetSymbolAddress of the scratch array: %s",
                           cudaGetErrorString(e));
    return TPA_ERR_CUDA;
  }
  return tpa_decode_attention(cache, q, q_pos, scale, out, max_len, splits, kernel, scratch, kNoAllocScratchBytes,
                              stream);
}
