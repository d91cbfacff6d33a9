// store_kv and gather_kv kernels.
//
// store_kv follows the pages' description of the scatter ("Mini-SGLang 完整剖析",
// §4.6.7: the attention backend first writes the step's K/V rows into the pool
// at out_loc; §4.9.4: rows of D elements with a row stride, int32 or int64
// indices, copied with 16-byte vectors).  Here every thread moves one 16-byte
// chunk of one row, so a warp covers 512 contiguous bytes of a row and the
// grid scales with the bytes moved rather than with the token count.
//
// gather_kv reads rows through the token-granular page table (§4.6.4) into a
// dense buffer; it is the translation the attention kernels do internally.
#include "common.cuh"
#include "launch.h"

namespace pkv {

__global__ void __launch_bounds__(256) store_kv_kernel(
    uint8_t* __restrict__ kpool, uint8_t* __restrict__ vpool, int64_t slot_stride_bytes,
    int64_t num_slots, const uint8_t* __restrict__ k, int64_t k_stride_bytes,
    const uint8_t* __restrict__ v, int64_t v_stride_bytes, const void* __restrict__ out_loc,
    int loc_i64, int64_t n, int32_t chunks_per_row, int32_t* err) {
  // The attention kernel that follows may start its set-up now; it waits for
  // this grid before it reads the pool.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t total = n * 2 * chunks_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / chunks_per_row;          // 0 .. 2n-1
    const int32_t chunk = static_cast<int32_t>(idx - row * chunks_per_row);
    const int64_t i = row >> 1;
    const bool is_v = row & 1;
    const int64_t slot = loc_i64 ? reinterpret_cast<const int64_t*>(out_loc)[i]
                                 : static_cast<int64_t>(reinterpret_cast<const int32_t*>(out_loc)[i]);
    if (slot < 0 || slot >= num_slots) {
      if (chunk == 0 && !is_v) set_err(err, PKV_DEV_ERR_SLOT_RANGE);
      continue;
    }
    const uint8_t* src = (is_v ? v + i * v_stride_bytes : k + i * k_stride_bytes) + chunk * 16;
    uint8_t* dst = (is_v ? vpool : kpool) + slot * slot_stride_bytes + chunk * 16;
    *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
  }
}

// FP8 pool: each thread turns 16 bf16 values (two 16-byte loads) into 16
// E4M3 codes of x * (1 / scale) and stores them as one 16-byte word.
__global__ void __launch_bounds__(256) store_kv_fp8_kernel(
    uint8_t* __restrict__ kpool, uint8_t* __restrict__ vpool, int64_t slot_stride_bytes,
    int64_t num_slots, const uint8_t* __restrict__ k, int64_t k_stride_bytes,
    const uint8_t* __restrict__ v, int64_t v_stride_bytes, const void* __restrict__ out_loc,
    int loc_i64, int64_t n, int32_t chunks_per_row, float k_inv, float v_inv, int32_t* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t total = n * 2 * chunks_per_row;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / chunks_per_row;
    const int32_t chunk = static_cast<int32_t>(idx - row * chunks_per_row);
    const int64_t i = row >> 1;
    const bool is_v = row & 1;
    const int64_t slot = loc_i64 ? reinterpret_cast<const int64_t*>(out_loc)[i]
                                 : static_cast<int64_t>(reinterpret_cast<const int32_t*>(out_loc)[i]);
    if (slot < 0 || slot >= num_slots) {
      if (chunk == 0 && !is_v) set_err(err, PKV_DEV_ERR_SLOT_RANGE);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>((is_v ? v + i * v_stride_bytes : k + i * k_stride_bytes) +
                                                      chunk * 32);
    const float inv = is_v ? v_inv : k_inv;
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t wa[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float f0[8], f1[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 p = bf16x2_to_f2(wa[e]), q = bf16x2_to_f2(wa[4 + e]);
      f0[2 * e] = p.x;
      f0[2 * e + 1] = p.y;
      f1[2 * e] = q.x;
      f1[2 * e + 1] = q.y;
    }
    const uint2 lo = quant8_e4m3(f0, inv), hi = quant8_e4m3(f1, inv);
    uint8_t* dst = (is_v ? vpool : kpool) + slot * slot_stride_bytes + chunk * 16;
    *reinterpret_cast<uint4*>(dst) = make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
}

cudaError_t launch_store_kv(const PoolView& pool, const void* k, int64_t k_stride_bytes,
                            const void* v, int64_t v_stride_bytes, const void* out_loc,
                            bool loc_i64, int64_t n, int32_t* err, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (pool.dtype == PKV_DTYPE_FP8_E4M3) {
    const int32_t cpr = pool.num_kv_heads * kHeadDim / 16;  // 16 codes per thread
    const int64_t total = n * 2 * cpr;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    // The inverse scales are float32 divisions, rounded to nearest.
    const float k_inv = 1.0f / pool.k_scale, v_inv = 1.0f / pool.v_scale;
    store_kv_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        pool.k_mut, pool.v_mut, pool.slot_stride_bytes, pool.num_slots,
        static_cast<const uint8_t*>(k), k_stride_bytes, static_cast<const uint8_t*>(v),
        v_stride_bytes, out_loc, loc_i64 ? 1 : 0, n, cpr, k_inv, v_inv, err);
    return cudaGetLastError();
  }
  const int32_t row_bytes = pool.num_kv_heads * kHeadDim * pool.esize;
  const int32_t cpr = row_bytes / 16;
  const int64_t total = n * 2 * cpr;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  store_kv_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      pool.k_mut, pool.v_mut, pool.slot_stride_bytes, pool.num_slots,
      static_cast<const uint8_t*>(k), k_stride_bytes, static_cast<const uint8_t*>(v),
      v_stride_bytes, out_loc, loc_i64 ? 1 : 0, n, cpr, err);
  return cudaGetLastError();
}

// One block column per request (blockIdx.y); warps stride over its tokens,
// each lane moving 16-byte chunks of the K and V rows.
__global__ void __launch_bounds__(256) gather_kv_kernel(
    const uint8_t* __restrict__ kpool, const uint8_t* __restrict__ vpool, int64_t slot_stride_bytes,
    int64_t num_slots, int32_t page_size, const int32_t* __restrict__ table, int64_t rows,
    int64_t cols, int64_t row_stride, const int32_t* __restrict__ table_idx,
    const int32_t* __restrict__ seq_lens, const int64_t* __restrict__ row_offsets,
    int32_t row_bytes, uint8_t* __restrict__ k_out, uint8_t* __restrict__ v_out, int32_t* err) {
  const int r = blockIdx.y;
  const int32_t tr = table_idx[r];
  int64_t n = seq_lens[r];
  const int64_t base = row_offsets[r];
  const bool row_ok = tr >= 0 && tr < rows;
  if (!row_ok && threadIdx.x == 0 && blockIdx.x == 0) set_err(err, PKV_DEV_ERR_TABLE_RANGE);
  if (n > cols) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_err(err, PKV_DEV_ERR_TABLE_RANGE);
  }
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cpr = row_bytes >> 4;
  for (int64_t j = blockIdx.x * warps + warp; j < n; j += (int64_t)gridDim.x * warps) {
    int64_t slot = -1;
    if (row_ok && j < cols) {
      if (lane == 0) slot = token_slot(table + tr * row_stride, j, page_size, num_slots, err);
      slot = __shfl_sync(0xffffffffu, slot, 0);
    }
    uint8_t* kd = k_out + (base + j) * row_bytes;
    uint8_t* vd = v_out + (base + j) * row_bytes;
    for (int c = lane; c < cpr; c += 32) {
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (slot >= 0) {
        kv = __ldg(reinterpret_cast<const uint4*>(kpool + slot * slot_stride_bytes) + c);
        vv = __ldg(reinterpret_cast<const uint4*>(vpool + slot * slot_stride_bytes) + c);
      }
      reinterpret_cast<uint4*>(kd)[c] = kv;
      reinterpret_cast<uint4*>(vd)[c] = vv;
    }
  }
}

cudaError_t launch_gather_kv(const PoolView& pool, const TableView& t, const int32_t* table_idx,
                             const int32_t* seq_lens, const int64_t* row_offsets, int32_t batch,
                             void* k_out, void* v_out, int32_t* err, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  const int32_t row_bytes = pool.num_kv_heads * kHeadDim * pool.esize;
  dim3 grid(16, batch);
  gather_kv_kernel<<<grid, 256, 0, s>>>(pool.k, pool.v, pool.slot_stride_bytes, pool.num_slots,
                                        pool.page_size, t.entries, t.rows, t.cols, t.row_stride,
                                        table_idx, seq_lens, row_offsets, row_bytes,
                                        static_cast<uint8_t*>(k_out), static_cast<uint8_t*>(v_out),
                                        err);
  return cudaGetLastError();
}

}  // namespace pkv
