// Host-side launchers of the pkv kernels (internal; the public ABI is include/pkv.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

constexpr int kHeadDimHost = 128;
constexpr int kMaxDevicesHost = 64;

// Raise `kernel`'s dynamic shared memory limit to `bytes` once per device.
// `state` is the caller's per-kernel array (one entry per device) of the
// limit already set, so calls after the first make no CUDA call at all (this
// keeps launches legal inside stream capture once the kernel has run once).
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel kernel, int bytes, int* state) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesHost) return cudaErrorInvalidDevice;
  if (state[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) state[dev] = bytes;
  return e;
}

// Driver entry point of cuTensorMapEncodeTiled (null when unavailable).
void* tensor_map_encode_fn();

struct PoolView {
  const uint8_t* k;  // layer base (bytes)
  const uint8_t* v;
  uint8_t* k_mut;
  uint8_t* v_mut;
  int64_t slot_stride_bytes;
  int64_t num_slots;
  int32_t num_kv_heads;
  int32_t page_size;
  int32_t esize;  // element size in bytes
  int32_t dtype;
  float k_scale, v_scale;  // FP8 dequantisation scales (1 otherwise)
};

struct TableView {
  const int32_t* entries;
  int64_t rows;
  int64_t cols;
  int64_t row_stride;
};

cudaError_t launch_store_kv(const PoolView& pool, const void* k, int64_t k_stride_bytes,
                            const void* v, int64_t v_stride_bytes, const void* out_loc,
                            bool loc_i64, int64_t n, int32_t* err, cudaStream_t s);

cudaError_t launch_qk_norm_rope_store(const PoolView& pool, const void* qkv, int64_t qkv_row_stride,
                                      int32_t num_q_heads, const void* positions, bool pos_i64,
                                      const float* cos_sin, int64_t max_position, const void* q_w,
                                      const void* k_w, float eps, const void* out_loc, bool loc_i64,
                                      int64_t n, void* q_out, int32_t* err, cudaStream_t s);

cudaError_t launch_wait_timeout(int32_t* err, cudaStream_t s);

cudaError_t launch_gather_kv(const PoolView& pool, const TableView& t, const int32_t* table_idx,
                             const int32_t* seq_lens, const int64_t* row_offsets, int32_t batch,
                             void* k_out, void* v_out, int32_t* err, cudaStream_t s);

// Split-KV decode.
size_t decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int grid);
int decode_grid_size();
// Cascade decode: the suffix pass's column offsets and the shared-prefix
// partials the combine kernel merges ([nsplit][batch][hq] (max, sum) pairs and
// [nsplit][batch][hq][128] fp32 rows).
struct CascadeView {
  const int32_t* kv_start;
  const float2* pre_ml;
  const float* pre_o;
  int32_t nsplit;
  // When set, the prefix pass runs on another stream: the merge kernel's
  // stream waits for this event (recorded after the prefix pass) first.
  cudaEvent_t prefix_done = nullptr;
};

cudaError_t launch_decode(const PoolView& pool, const TableView& t, const void* q,
                          int32_t num_q_heads, const int32_t* table_idx, const int32_t* seq_lens,
                          int32_t batch, float scale, void* out, void* workspace, int grid,
                          int32_t* err, cudaStream_t s,
                          const struct CascadeView* cascade = nullptr);

// Extend: tcgen05 path (bf16) and CUDA-core path (fp32 check build).
cudaError_t launch_extend_tc(const PoolView& pool, const TableView& t, const void* q,
                             int32_t num_q_heads, const int32_t* table_idx,
                             const int32_t* prefix_lens, const int32_t* extend_lens,
                             const int32_t* q_offsets, int32_t batch, int64_t total_q, int32_t max_extend,
                             float scale, void* out, int32_t* err, cudaStream_t s);

cudaError_t launch_extend_prefix(const PoolView& pool, const TableView& t, const void* q,
                                 int32_t num_q_heads, const int32_t* table_idx,
                                 const int32_t* group_offsets, const int32_t* group_prefix,
                                 int32_t num_groups, int32_t batch, int32_t nsplit, int32_t split_keys,
                                 float scale, float2* pre_ml, float* pre_o, int32_t* err, cudaStream_t s);

cudaError_t launch_cascade_prep(const int32_t* group_offsets, const int32_t* group_prefix,
                                int32_t num_groups, const int32_t* seq_lens, int32_t batch,
                                int64_t prefix_capacity, int32_t* kv_start, int32_t* err,
                                cudaStream_t s);

size_t cascade_workspace_bytes(int32_t batch, int32_t num_q_heads, int64_t max_prefix_len);

cudaError_t launch_decode_cascade(const PoolView& pool, const TableView& t, const void* q,
                                  int32_t num_q_heads, const int32_t* table_idx,
                                  const int32_t* seq_lens, int32_t batch,
                                  const int32_t* group_offsets, const int32_t* group_prefix,
                                  int32_t num_groups, int64_t max_prefix_len, float scale, void* out,
                                  void* workspace, int32_t* err, cudaStream_t s);
cudaError_t launch_extend_simt(const PoolView& pool, const TableView& t, const void* q,
                               int32_t num_q_heads, const int32_t* table_idx,
                               const int32_t* prefix_lens, const int32_t* extend_lens,
                               const int32_t* q_offsets, int32_t batch, int64_t total_q, int32_t max_extend,
                               float scale, void* out, int32_t* err, cudaStream_t s);

}  // namespace pkv
