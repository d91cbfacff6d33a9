// Library-owned workspace objects: the one place the library allocates.
//
// A caller that prefers not to size and own scratch memory creates one
// workspace per stream at start-up (before any graph capture), passes its
// buffer to decode / cascade decode / extend, and its error word as dev_err;
// pkv_read_device_error synchronises the stream, returns the accumulated
// pkv_device_error bits and clears them.
#include <cuda_runtime.h>

#include <new>

#include "launch.h"

struct pkv_workspace {
  void* buf;
  size_t bytes;
  int32_t* err;
  int device;
};

extern "C" {

int pkv_workspace_create(int32_t max_batch, int32_t max_q_heads, int64_t max_prefix_len,
                         pkv_workspace** out) {
  if (out == nullptr) return PKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (max_batch < 1 || max_q_heads < 1 || max_prefix_len < 0) return PKV_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  const int grid = pkv::decode_grid_size();
  size_t bytes = pkv::decode_workspace_bytes(max_batch, max_q_heads, grid);
  const size_t cas = pkv::cascade_workspace_bytes(max_batch, max_q_heads, max_prefix_len);
  if (cas > bytes) bytes = cas;
  pkv_workspace* ws = new (std::nothrow) pkv_workspace{nullptr, bytes, nullptr, dev};
  if (ws == nullptr) return PKV_ERR_INVALID_ARG;
  if (cudaMalloc(&ws->buf, bytes) != cudaSuccess || cudaMalloc(&ws->err, sizeof(int32_t)) != cudaSuccess ||
      cudaMemset(ws->err, 0, sizeof(int32_t)) != cudaSuccess) {
    cudaFree(ws->buf);
    cudaFree(ws->err);
    delete ws;
    return PKV_ERR_CUDA;
  }
  *out = ws;
  return PKV_OK;
}

void pkv_workspace_destroy(pkv_workspace* ws) {
  if (ws == nullptr) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(ws->device);
  cudaFree(ws->buf);
  cudaFree(ws->err);
  cudaSetDevice(prev);
  delete ws;
}

void* pkv_workspace_buffer(const pkv_workspace* ws, size_t* bytes) {
  if (ws == nullptr) {
    if (bytes) *bytes = 0;
    return nullptr;
  }
  if (bytes) *bytes = ws->bytes;
  return ws->buf;
}

int32_t* pkv_workspace_error_word(const pkv_workspace* ws) { return ws ? ws->err : nullptr; }

int pkv_read_device_error(pkv_workspace* ws, pkv_stream_t stream, int32_t* code) {
  if (ws == nullptr || code == nullptr) return PKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, ws->err, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(ws->err, 0, sizeof(int32_t), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return PKV_ERR_CUDA;
  *code = h;
  return PKV_OK;
}

}  // extern "C"
