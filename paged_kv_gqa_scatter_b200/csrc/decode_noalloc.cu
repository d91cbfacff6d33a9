// pkv_decode_attn_noalloc: split-KV decode whose scratch lives in a fixed
// device array owned by this library, for callers that cannot allocate.
//
// Who needs it: a serving engine that hands nearly all free device memory to
// its KV pool at start-up (the pool is sized from the memory left after the
// weights) has no headroom to allocate a workspace later, and code running
// inside a host framework that owns every device allocation (a plugin or FFI
// host) may have no allocator handle at all.  Such callers pass only inputs and
// outputs; the partial results go to `g_decode_scratch` below.
//
// Properties a caller must know:
//  * The array is kNoAllocScratchBytes (16 MiB) on every device that loads the
//    library, held until the process exits.
//  * Host code cannot use the array's name as a device address.  Every call
//    made outside stream capture (with its device current) looks the address
//    up with cudaGetSymbolAddress and caches it per device, so a device reset
//    that reloads the library's device code is picked up by the next such
//    call.  A call made while its stream is being captured uses the cached
//    address (or looks it up if there is none yet); make the first call on a
//    device outside any stream capture, and make another one after a device
//    reset before capturing again.
//  * Every call on a device shares the one array, so calls that may overlap on
//    the GPU (different streams without ordering between them) race and can
//    corrupt each other's results.  Calls ordered on one stream are safe.
//  * Nothing in the array has to start at zero: every byte a call reads was
//    written earlier in the same call, so leftover contents of the previous call
//    are harmless.
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device.  Looked up again
// on every call that is not being captured; a call under capture reuses the
// address cached by the last uncaptured call.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (cs == cudaStreamCaptureStatusNone || g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return PKV_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PKV_OK;
}

}  // namespace

extern "C" {

size_t pkv_decode_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

int pkv_decode_attn_noalloc(const pkv_pool* pool, int32_t layer, const void* q, int32_t num_q_heads,
                            const pkv_page_table* table, const int32_t* table_idx,
                            const int32_t* seq_lens, int32_t batch, float scale, void* out,
                            int32_t* dev_err, pkv_stream_t stream) {
  if (batch < 0 || num_q_heads < 1) return PKV_ERR_INVALID_ARG;
  if (pkv_decode_workspace_bytes(batch, num_q_heads) > kNoAllocScratchBytes) return PKV_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (st != PKV_OK) return st;
  return pkv_decode_attn(pool, layer, q, num_q_heads, table, table_idx, seq_lens, batch, scale, out,
                         scratch, kNoAllocScratchBytes, dev_err, stream);
}

}  // extern "C"
