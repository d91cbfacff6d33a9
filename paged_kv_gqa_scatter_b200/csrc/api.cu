// extern "C" entry points declared in include/pkv.h: argument checks, then launches.
//
// The checks mirror the declarative shape/dtype/stride checks the pages
// describe for the upstream store kernel ("Mini-SGLang 完整剖析" §4.9.4:
// every tensor is matched against symbolic sizes, strides and dtypes before
// launch and a failure reports where it happened); here a failure returns a
// pkv_status before anything is launched.
#include <cuda_runtime.h>

#include <climits>

#include "launch.h"

using pkv::PoolView;
using pkv::TableView;

namespace {

constexpr int kMaxDecodeBatch = 4096;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int esize_of(int32_t dtype) {
  if (dtype == PKV_DTYPE_BF16) return 2;
  if (dtype == PKV_DTYPE_F32) return 4;
  if (dtype == PKV_DTYPE_FP8_E4M3) return 1;
  return 0;
}

// Element size of the rows a call reads or writes beside the pool (k/v to
// store, qkv, q, out): bf16 for an FP8 pool, the pool's type otherwise.
int io_esize(const PoolView& pv) { return pv.dtype == PKV_DTYPE_FP8_E4M3 ? 2 : pv.esize; }

bool finite_positive(float x) { return x > 0.f && x <= 3.402823466e38f; }

int check_pool(const pkv_pool* p, int32_t layer, PoolView* out) {
  if (p == nullptr || p->k == nullptr || p->v == nullptr) return PKV_ERR_INVALID_ARG;
  const int es = esize_of(p->dtype);
  if (es == 0) return PKV_ERR_UNSUPPORTED;
  if (p->head_dim != pkv::kHeadDimHost) return PKV_ERR_UNSUPPORTED;
  if (p->num_kv_heads < 1 || p->num_layers < 1 || p->num_slots < 1 || p->page_size < 1)
    return PKV_ERR_INVALID_ARG;
  if (layer < 0 || layer >= p->num_layers) return PKV_ERR_INVALID_ARG;
  if (p->dtype == PKV_DTYPE_FP8_E4M3 && !(finite_positive(p->k_scale) && finite_positive(p->v_scale)))
    return PKV_ERR_INVALID_ARG;
  const int64_t row = static_cast<int64_t>(p->num_kv_heads) * p->head_dim;
  if (p->slot_stride < row || p->layer_stride < 0) return PKV_ERR_INVALID_ARG;
  if (p->num_layers > 1 && p->layer_stride < p->num_slots * p->slot_stride) return PKV_ERR_INVALID_ARG;
  if (p->num_slots % p->page_size != 0) return PKV_ERR_INVALID_ARG;
  if (!aligned16(p->k) || !aligned16(p->v)) return PKV_ERR_MISALIGNED;
  if ((p->slot_stride * es) % 16 != 0 || (p->layer_stride * es) % 16 != 0) return PKV_ERR_MISALIGNED;
  const int64_t layer_off = static_cast<int64_t>(layer) * p->layer_stride * es;
  out->k = static_cast<const uint8_t*>(p->k) + layer_off;
  out->v = static_cast<const uint8_t*>(p->v) + layer_off;
  out->k_mut = static_cast<uint8_t*>(p->k) + layer_off;
  out->v_mut = static_cast<uint8_t*>(p->v) + layer_off;
  out->slot_stride_bytes = p->slot_stride * es;
  out->num_slots = p->num_slots;
  out->num_kv_heads = p->num_kv_heads;
  out->page_size = p->page_size;
  out->esize = es;
  out->dtype = p->dtype;
  out->k_scale = p->dtype == PKV_DTYPE_FP8_E4M3 ? p->k_scale : 1.f;
  out->v_scale = p->dtype == PKV_DTYPE_FP8_E4M3 ? p->v_scale : 1.f;
  return PKV_OK;
}

int check_table(const pkv_page_table* t, TableView* out) {
  if (t == nullptr || t->entries == nullptr) return PKV_ERR_INVALID_ARG;
  if (t->rows < 1 || t->cols < 1 || t->row_stride < t->cols) return PKV_ERR_INVALID_ARG;
  if (t->cols > INT_MAX) return PKV_ERR_TOO_LARGE;
  out->entries = t->entries;
  out->rows = t->rows;
  out->cols = t->cols;
  out->row_stride = t->row_stride;
  return PKV_OK;
}

// Head counts: Hkv <= 8 and G = Hq / Hkv in {1, 2, 4, 8}; plain decode on a
// bf16 or E4M3 pool also takes G = 16 (two 8-head column tiles).
int check_heads(const pkv_pool* p, int32_t num_q_heads, bool group16_ok = false) {
  if (p->num_kv_heads > 8) return PKV_ERR_UNSUPPORTED;
  if (num_q_heads < 1 || num_q_heads % p->num_kv_heads != 0) return PKV_ERR_INVALID_ARG;
  const int G = num_q_heads / p->num_kv_heads;
  if (G == 16 && group16_ok && p->dtype != PKV_DTYPE_F32) return PKV_OK;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PKV_ERR_UNSUPPORTED;
  return PKV_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA; }

}  // namespace

extern "C" {

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported dtype, head_dim or head counts";
    case PKV_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case PKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PKV_ERR_CUDA: return "CUDA runtime error";
    case PKV_ERR_TOO_LARGE: return "size beyond a documented maximum";
    default: return "unknown status";
  }
}

const char* pkv_version(void) { return "pkv 0.1 sm_100a"; }

int pkv_store_kv(const pkv_pool* pool, int32_t layer, const void* k, int64_t k_row_stride,
                 const void* v, int64_t v_row_stride, const void* out_loc,
                 int32_t out_loc_is_i64, int64_t n_tokens, int32_t* dev_err,
                 pkv_stream_t stream) {
  PoolView pv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  if (n_tokens < 0) return PKV_ERR_INVALID_ARG;
  if (n_tokens == 0) return PKV_OK;
  if (k == nullptr || v == nullptr || out_loc == nullptr) return PKV_ERR_INVALID_ARG;
  const int64_t row = static_cast<int64_t>(pool->num_kv_heads) * pool->head_dim;
  if (k_row_stride < row || v_row_stride < row) return PKV_ERR_INVALID_ARG;
  if (out_loc_is_i64 != 0 && out_loc_is_i64 != 1) return PKV_ERR_INVALID_ARG;
  const int ies = io_esize(pv);
  if (!aligned16(k) || !aligned16(v) || (k_row_stride * ies) % 16 != 0 ||
      (v_row_stride * ies) % 16 != 0)
    return PKV_ERR_MISALIGNED;
  return from_cuda(pkv::launch_store_kv(pv, k, k_row_stride * ies, v, v_row_stride * ies,
                                        out_loc, out_loc_is_i64 == 1, n_tokens, dev_err,
                                        static_cast<cudaStream_t>(stream)));
}

int pkv_qk_norm_rope_store(const pkv_pool* pool, int32_t layer, const void* qkv,
                           int64_t qkv_row_stride, int32_t num_q_heads, const void* positions,
                           int32_t positions_is_i64, const float* cos_sin_cache,
                           int64_t max_position, const void* q_norm_weight,
                           const void* k_norm_weight, float eps, const void* out_loc,
                           int32_t out_loc_is_i64, int64_t n_tokens, void* q_out,
                           int32_t* dev_err, pkv_stream_t stream) {
  PoolView pv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  if (n_tokens < 0 || max_position < 1) return PKV_ERR_INVALID_ARG;
  if (n_tokens == 0) return PKV_OK;
  if (num_q_heads < 1) return PKV_ERR_INVALID_ARG;
  if (!qkv || !positions || !cos_sin_cache || !out_loc || !q_out) return PKV_ERR_INVALID_ARG;
  if (positions_is_i64 != 0 && positions_is_i64 != 1) return PKV_ERR_INVALID_ARG;
  if (out_loc_is_i64 != 0 && out_loc_is_i64 != 1) return PKV_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return PKV_ERR_INVALID_ARG;
  const int64_t row = static_cast<int64_t>(num_q_heads + 2 * pool->num_kv_heads) * pool->head_dim;
  if (qkv_row_stride < row) return PKV_ERR_INVALID_ARG;
  if (!aligned16(qkv) || (qkv_row_stride * io_esize(pv)) % 16 != 0 || !aligned16(q_out) ||
      !aligned16(cos_sin_cache) || (q_norm_weight && !aligned16(q_norm_weight)) ||
      (k_norm_weight && !aligned16(k_norm_weight)))
    return PKV_ERR_MISALIGNED;
  return from_cuda(pkv::launch_qk_norm_rope_store(
      pv, qkv, qkv_row_stride, num_q_heads, positions, positions_is_i64 == 1, cos_sin_cache,
      max_position, q_norm_weight, k_norm_weight, eps, out_loc, out_loc_is_i64 == 1, n_tokens,
      q_out, dev_err, static_cast<cudaStream_t>(stream)));
}

int pkv_selftest_wait_timeout(int32_t* dev_err, pkv_stream_t stream) {
  if (dev_err == nullptr) return PKV_ERR_INVALID_ARG;
  return from_cuda(pkv::launch_wait_timeout(dev_err, static_cast<cudaStream_t>(stream)));
}

int pkv_gather_kv(const pkv_pool* pool, int32_t layer, const pkv_page_table* table,
                  const int32_t* table_idx, const int32_t* seq_lens, const int64_t* row_offsets,
                  int32_t batch, void* k_out, void* v_out, int32_t* dev_err,
                  pkv_stream_t stream) {
  PoolView pv;
  TableView tv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  if (batch < 0) return PKV_ERR_INVALID_ARG;
  if (batch == 0) return PKV_OK;
  if (batch > 65535) return PKV_ERR_TOO_LARGE;
  st = check_table(table, &tv);
  if (st != PKV_OK) return st;
  if (!table_idx || !seq_lens || !row_offsets || !k_out || !v_out) return PKV_ERR_INVALID_ARG;
  if (!aligned16(k_out) || !aligned16(v_out)) return PKV_ERR_MISALIGNED;
  return from_cuda(pkv::launch_gather_kv(pv, tv, table_idx, seq_lens, row_offsets, batch, k_out,
                                         v_out, dev_err, static_cast<cudaStream_t>(stream)));
}

size_t pkv_decode_workspace_bytes(int32_t batch, int32_t num_q_heads) {
  if (batch < 0 || num_q_heads < 1) return 0;
  return pkv::decode_workspace_bytes(batch, num_q_heads, pkv::decode_grid_size());
}

int pkv_decode_attn(const pkv_pool* pool, int32_t layer, const void* q, int32_t num_q_heads,
                    const pkv_page_table* table, const int32_t* table_idx,
                    const int32_t* seq_lens, int32_t batch, float scale, void* out,
                    void* workspace, size_t workspace_bytes, int32_t* dev_err,
                    pkv_stream_t stream) {
  PoolView pv;
  TableView tv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  st = check_heads(pool, num_q_heads, /*group16_ok=*/true);
  if (st != PKV_OK) return st;
  if (batch < 0) return PKV_ERR_INVALID_ARG;
  if (batch == 0) return PKV_OK;
  if (batch > kMaxDecodeBatch) return PKV_ERR_TOO_LARGE;
  st = check_table(table, &tv);
  if (st != PKV_OK) return st;
  if (static_cast<int64_t>(batch) * tv.cols > INT_MAX) return PKV_ERR_TOO_LARGE;
  if (!q || !out || !table_idx || !seq_lens) return PKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return PKV_ERR_MISALIGNED;
  const int grid = pkv::decode_grid_size();
  const size_t need = pkv::decode_workspace_bytes(batch, num_q_heads, grid);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  return from_cuda(pkv::launch_decode(pv, tv, q, num_q_heads, table_idx, seq_lens, batch, scale,
                                      out, workspace, grid, dev_err,
                                      static_cast<cudaStream_t>(stream)));
}

size_t pkv_decode_cascade_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                          int64_t max_prefix_len) {
  if (batch < 0 || num_q_heads < 1 || max_prefix_len < 0) return 0;
  return pkv::cascade_workspace_bytes(batch, num_q_heads, max_prefix_len);
}

int pkv_decode_attn_cascade(const pkv_pool* pool, int32_t layer, const void* q,
                            int32_t num_q_heads, const pkv_page_table* table,
                            const int32_t* table_idx, const int32_t* seq_lens, int32_t batch,
                            const int32_t* group_offsets, const int32_t* group_prefix_lens,
                            int32_t num_groups, int64_t max_prefix_len, float scale, void* out,
                            void* workspace, size_t workspace_bytes, int32_t* dev_err,
                            pkv_stream_t stream) {
  PoolView pv;
  TableView tv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  if (pv.dtype == PKV_DTYPE_F32) return PKV_ERR_UNSUPPORTED;
  st = check_heads(pool, num_q_heads);
  if (st != PKV_OK) return st;
  if (batch < 0 || num_groups < 0 || max_prefix_len < 0) return PKV_ERR_INVALID_ARG;
  if (batch == 0) return PKV_OK;
  if (num_groups < 1 || num_groups > batch) return PKV_ERR_INVALID_ARG;
  if (batch > kMaxDecodeBatch) return PKV_ERR_TOO_LARGE;
  st = check_table(table, &tv);
  if (st != PKV_OK) return st;
  if (static_cast<int64_t>(batch) * tv.cols > INT_MAX || max_prefix_len > tv.cols) return PKV_ERR_TOO_LARGE;
  if (!q || !out || !table_idx || !seq_lens || !group_offsets || !group_prefix_lens)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return PKV_ERR_MISALIGNED;
  const size_t need = pkv::cascade_workspace_bytes(batch, num_q_heads, max_prefix_len);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  return from_cuda(pkv::launch_decode_cascade(pv, tv, q, num_q_heads, table_idx, seq_lens, batch,
                                              group_offsets, group_prefix_lens, num_groups,
                                              max_prefix_len, scale, out, workspace, dev_err,
                                              static_cast<cudaStream_t>(stream)));
}

size_t pkv_extend_workspace_bytes(int32_t batch, int32_t num_q_heads, int64_t total_q) {
  (void)batch;
  (void)num_q_heads;
  (void)total_q;
  return 0;
}

int pkv_extend_attn(const pkv_pool* pool, int32_t layer, const void* q, int32_t num_q_heads,
                    const pkv_page_table* table, const int32_t* table_idx,
                    const int32_t* prefix_lens, const int32_t* extend_lens,
                    const int32_t* q_offsets, int32_t batch, int64_t total_q,
                    int32_t max_extend_len, float scale, void* out, void* workspace,
                    size_t workspace_bytes, int32_t* dev_err, pkv_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  PoolView pv;
  TableView tv;
  int st = check_pool(pool, layer, &pv);
  if (st != PKV_OK) return st;
  st = check_heads(pool, num_q_heads);
  if (st != PKV_OK) return st;
  if (batch < 0 || total_q < 0 || max_extend_len < 0) return PKV_ERR_INVALID_ARG;
  if (batch == 0 || total_q == 0 || max_extend_len == 0) return PKV_OK;
  if (batch > 65535) return PKV_ERR_TOO_LARGE;
  st = check_table(table, &tv);
  if (st != PKV_OK) return st;
  if (!q || !out || !table_idx || !prefix_lens || !extend_lens || !q_offsets)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return PKV_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pv.dtype == PKV_DTYPE_BF16 || pv.dtype == PKV_DTYPE_FP8_E4M3)
    return from_cuda(pkv::launch_extend_tc(pv, tv, q, num_q_heads, table_idx, prefix_lens,
                                           extend_lens, q_offsets, batch, total_q, max_extend_len, scale,
                                           out, dev_err, s));
  return from_cuda(pkv::launch_extend_simt(pv, tv, q, num_q_heads, table_idx, prefix_lens,
                                           extend_lens, q_offsets, batch, total_q, max_extend_len, scale,
                                           out, dev_err, s));
}

}  // extern "C"
