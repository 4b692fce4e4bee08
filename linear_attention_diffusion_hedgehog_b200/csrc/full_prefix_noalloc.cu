// Allocation-free entry point for the softmax teacher: bha_full_prefix_attn with its split
// scratch taken from a fixed array that lives in the library's own device image.
//
// Who needs it: callers that must not allocate device memory on the call path, such as a
// serving engine that reserves the whole GPU memory budget up front (weights plus a fixed
// cache pool) and forbids cudaMalloc inside its decode loop, or a plugin embedded in a host
// that owns all allocation and gives it no allocator.  They still pass Q, the caches and O;
// only the split partials move into library-owned memory.
//
// The scratch is a file-scope __device__ array of BHA_NOALLOC_SCRATCH_BYTES; every GPU that
// loads the library holds one copy until the process exits.  Host code cannot pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so the first call on
// each device, with that device current, looks up its device address once with
// cudaGetSymbolAddress and every later call on that device reuses it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bha.h"

namespace {

__device__ __align__(256) unsigned char g_full_prefix_scratch[BHA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of this device's copy of the scratch array (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BHA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BHA_ERR_UNSUPPORTED;
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_full_prefix_scratch);
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch_ptr[dev] == nullptr) return BHA_ERR_CUDA;
  *out = g_scratch_ptr[dev];
  return BHA_OK;
}

}  // namespace

extern "C" int bha_full_prefix_attn_noalloc(const bha_dims* dims, const int32_t* cu_blk,
                                            const int32_t* kv_len, const void* Q, const void* Kc,
                                            const void* Vc, int64_t kv_capacity, void* O,
                                            int32_t* dev_err, void* stream) {
  if (dims == nullptr) return BHA_ERR_INVALID;
  // Same split plan, hence the same scratch need, as bha_full_prefix_attn; a call that would
  // need more than the fixed array is refused before anything is launched.
  const size_t need = bha_full_prefix_workspace_bytes(dims, kv_capacity);
  if (need > (size_t)BHA_NOALLOC_SCRATCH_BYTES) return BHA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (need > 0) {
    const int s = scratch_address(&ws);
    if (s != BHA_OK) return s;
  }
  // Nothing in the scratch has to start at zero: every split writes each partial row that
  // the combine step later reads, so the previous call's contents are never consumed.
  return bha_full_prefix_attn(dims, cu_blk, kv_len, Q, Kc, Vc, kv_capacity, O, ws, need, dev_err,
                              stream);
}
