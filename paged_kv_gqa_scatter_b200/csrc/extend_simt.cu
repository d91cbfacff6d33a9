// Causal extend attention on CUDA cores (fp32 check build).
//
// What it computes: "深入解析 mini-sglang" (yunpan.plus), chunked prefill -- a
// chunk attends to the KV its request's earlier chunks left in the pool (same
// page-table row) plus its own rows; "Mini-SGLang 完整剖析" §4.2.3 -- the chunk
// holds extend_len = device_len - cached_len tokens after a cached prefix that
// may be shared through the radix cache (§1.4).  Query i of a chunk sits at
// position prefix + i and sees keys 0 .. prefix + i.
//
// Layout: one CTA per (query block, KV head, request); a block holds 64 query
// rows = 64/G tokens x the G query heads of that KV head.  Keys stream through
// shared memory in tiles of 32 (widened to fp32, K rows padded to 129 floats so
// that lane = key reads conflict-free); each warp owns 16 rows and keeps their
// online-softmax state (log2 domain) in registers.
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

constexpr int kRows = 64;
constexpr int kKeyTile = 32;
constexpr int kThreads = 128;
constexpr int kKPad = kHeadDim + 1;
// q rows, V tile, padded K tile, then the tile's slots (8-byte aligned).
constexpr int kSmemBytes = 4 * ((kRows + kKeyTile) * kHeadDim + kKeyTile * kKPad) + 8 * kKeyTile;
static_assert(((kRows + kKeyTile) * kHeadDim + kKeyTile * kKPad) % 2 == 0, "slots must be 8-byte aligned");

struct ExtendArgs {
  const uint8_t* kbase;
  const uint8_t* vbase;
  int64_t slot_stride_bytes;
  int64_t num_slots;
  const int32_t* table;
  int64_t table_rows, table_cols, table_stride;
  int32_t page_size;
  const int32_t* table_idx;
  const int32_t* prefix_lens;
  const int32_t* extend_lens;
  const int32_t* q_offsets;
  const void* q;
  void* out;
  int64_t total_q;
  int32_t max_extend;
  int32_t hq;
  float scale_log2;
  int32_t* err;
};

template <typename E>
__device__ __forceinline__ float to_f(E x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename E, int G>
__global__ void __launch_bounds__(kThreads) extend_simt_kernel(const ExtendArgs a) {
  constexpr int QB = kRows / G;          // query tokens per block
  constexpr int RPW = kRows / (kThreads / 32);  // rows per warp
  extern __shared__ __align__(16) float dyn[];
  float (*qs)[kHeadDim] = reinterpret_cast<float (*)[kHeadDim]>(dyn);
  float (*vs)[kHeadDim] = reinterpret_cast<float (*)[kHeadDim]>(dyn + kRows * kHeadDim);
  float (*ks)[kKPad] = reinterpret_cast<float (*)[kKPad]>(dyn + (kRows + kKeyTile) * kHeadDim);
  int64_t* slots = reinterpret_cast<int64_t*>(dyn + (kRows + kKeyTile) * kHeadDim + kKeyTile * kKPad);

  const int r = blockIdx.z, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t p = a.prefix_lens[r], e = a.extend_lens[r];
  if (p < 0 || e < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) set_err(a.err, PKV_DEV_ERR_BAD_LENGTH);
    return;
  }
  const int64_t qbase = a.q_offsets[r];
  if (qbase < 0 || qbase + e > a.total_q || e > a.max_extend) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) set_err(a.err, PKV_DEV_ERR_BAD_LENGTH);
    if (qbase < 0 || qbase + e > a.total_q) return;
  }
  const int i0 = blockIdx.x * QB;
  if (i0 >= e) return;
  const int32_t trow = a.table_idx[r];
  const bool row_ok = trow >= 0 && trow < a.table_rows;
  if (!row_ok && threadIdx.x == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
  int64_t kv_end = static_cast<int64_t>(p) + min(e, i0 + QB);
  if (kv_end > a.table_cols) {
    if (threadIdx.x == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
    kv_end = a.table_cols;
  }
  const int32_t* rowp = a.table + (row_ok ? trow : 0) * a.table_stride;
  const E* qg = static_cast<const E*>(a.q);

  // Query rows (token-major, then head), pre-scaled into the log2 domain.
  for (int idx = threadIdx.x; idx < kRows * kHeadDim; idx += kThreads) {
    const int row = idx / kHeadDim, d = idx % kHeadDim;
    const int tq = row / G, hh = row % G;
    const int i = i0 + tq;
    float x = 0.f;
    if (i < e) x = to_f<E>(qg[((qbase + i) * a.hq + g * G + hh) * kHeadDim + d]) * a.scale_log2;
    qs[row][d] = x;
  }

  float m[RPW], l[RPW], o[RPW][4];
#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    m[k] = -INFINITY;
    l[k] = 0.f;
    o[k][0] = o[k][1] = o[k][2] = o[k][3] = 0.f;
  }

  for (int64_t kt = 0; kt < kv_end; kt += kKeyTile) {
    __syncthreads();
    if (threadIdx.x < kKeyTile) {
      const int64_t j = kt + threadIdx.x;
      int64_t s = -1;
      if (j < kv_end && row_ok) s = token_slot(rowp, j, a.page_size, a.num_slots, a.err);
      slots[threadIdx.x] = s;
    }
    __syncthreads();
    {
      const int key = threadIdx.x / 4, part = threadIdx.x % 4;
      const int64_t s = slots[key];
      const E* kr = reinterpret_cast<const E*>(a.kbase + s * a.slot_stride_bytes) + g * kHeadDim;
      const E* vr = reinterpret_cast<const E*>(a.vbase + s * a.slot_stride_bytes) + g * kHeadDim;
      for (int d = part * 32; d < part * 32 + 32; ++d) {
        ks[key][d] = s >= 0 ? to_f<E>(kr[d]) : 0.f;
        vs[key][d] = s >= 0 ? to_f<E>(vr[d]) : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int row = warp * RPW + k;
      const int tq = row / G;
      const int i = i0 + tq;
      if (i >= e) continue;
      const int64_t lim = static_cast<int64_t>(p) + i + 1;  // keys < lim are visible
      if (kt >= lim) continue;
      const int64_t key = kt + lane;
      float sc = -INFINITY;
      if (key < lim && key < kv_end) {
        float acc = 0.f;
#pragma unroll 8
        for (int d = 0; d < kHeadDim; d += 4) {
          const float4 qv = *reinterpret_cast<const float4*>(&qs[row][d]);
          acc = fmaf(qv.x, ks[lane][d], acc);
          acc = fmaf(qv.y, ks[lane][d + 1], acc);
          acc = fmaf(qv.z, ks[lane][d + 2], acc);
          acc = fmaf(qv.w, ks[lane][d + 3], acc);
        }
        sc = acc;
      }
      float mx = sc;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[k], mx);
      const float alpha = exp2f(m[k] - mn);
      const float pk = exp2f(sc - mn);
      float ps = pk;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[k] = l[k] * alpha + ps;
      float o0 = o[k][0] * alpha, o1 = o[k][1] * alpha, o2 = o[k][2] * alpha, o3 = o[k][3] * alpha;
#pragma unroll 8
      for (int kk = 0; kk < kKeyTile; ++kk) {
        const float pb = __shfl_sync(0xffffffffu, pk, kk);
        const float4 vv = *reinterpret_cast<const float4*>(&vs[kk][4 * lane]);
        o0 = fmaf(pb, vv.x, o0);
        o1 = fmaf(pb, vv.y, o1);
        o2 = fmaf(pb, vv.z, o2);
        o3 = fmaf(pb, vv.w, o3);
      }
      o[k][0] = o0; o[k][1] = o1; o[k][2] = o2; o[k][3] = o3;
      m[k] = mn;
    }
  }

  E* og = static_cast<E*>(a.out);
#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    const int row = warp * RPW + k;
    const int tq = row / G, hh = row % G;
    const int i = i0 + tq;
    if (i >= e) continue;
    const float inv = l[k] > 0.f ? 1.f / l[k] : 0.f;
    E* dst = og + ((qbase + i) * a.hq + g * G + hh) * kHeadDim + 4 * lane;
    if constexpr (sizeof(E) == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(o[k][0] * inv, o[k][1] * inv, o[k][2] * inv, o[k][3] * inv);
    } else {
      uint2 w;
      w.x = pack_bf16x2(o[k][0] * inv, o[k][1] * inv);
      w.y = pack_bf16x2(o[k][2] * inv, o[k][3] * inv);
      *reinterpret_cast<uint2*>(dst) = w;
    }
  }
}

template <typename E, int G>
cudaError_t launch_t(const ExtendArgs& a, int hkv, int32_t batch, int32_t max_extend, cudaStream_t s) {
  constexpr int QB = kRows / G;
  dim3 grid((max_extend + QB - 1) / QB, hkv, batch);
  static int smem_state[kMaxDevicesHost] = {};
  cudaError_t err = ensure_smem_limit(extend_simt_kernel<E, G>, kSmemBytes, smem_state);
  if (err != cudaSuccess) return err;
  extend_simt_kernel<E, G><<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_extend_simt(const PoolView& pool, const TableView& t, const void* q,
                               int32_t num_q_heads, const int32_t* table_idx,
                               const int32_t* prefix_lens, const int32_t* extend_lens,
                               const int32_t* q_offsets, int32_t batch, int64_t total_q,
                               int32_t max_extend, float scale, void* out, int32_t* err,
                               cudaStream_t s) {
  if (batch == 0 || max_extend == 0) return cudaSuccess;
  ExtendArgs a;
  a.kbase = pool.k;
  a.vbase = pool.v;
  a.slot_stride_bytes = pool.slot_stride_bytes;
  a.num_slots = pool.num_slots;
  a.table = t.entries;
  a.table_rows = t.rows;
  a.table_cols = t.cols;
  a.table_stride = t.row_stride;
  a.page_size = pool.page_size;
  a.table_idx = table_idx;
  a.prefix_lens = prefix_lens;
  a.extend_lens = extend_lens;
  a.q_offsets = q_offsets;
  a.q = q;
  a.out = out;
  a.total_q = total_q;
  a.max_extend = max_extend;
  a.hq = num_q_heads;
  a.scale_log2 = scale * kLog2e;
  a.err = err;
  const int G = num_q_heads / pool.num_kv_heads;
  const int hkv = pool.num_kv_heads;
  if (pool.dtype == PKV_DTYPE_F32) {
    switch (G) {
      case 1: return launch_t<float, 1>(a, hkv, batch, max_extend, s);
      case 2: return launch_t<float, 2>(a, hkv, batch, max_extend, s);
      case 4: return launch_t<float, 4>(a, hkv, batch, max_extend, s);
      case 8: return launch_t<float, 8>(a, hkv, batch, max_extend, s);
    }
  } else {
    switch (G) {
      case 1: return launch_t<__nv_bfloat16, 1>(a, hkv, batch, max_extend, s);
      case 2: return launch_t<__nv_bfloat16, 2>(a, hkv, batch, max_extend, s);
      case 4: return launch_t<__nv_bfloat16, 4>(a, hkv, batch, max_extend, s);
      case 8: return launch_t<__nv_bfloat16, 8>(a, hkv, batch, max_extend, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace pkv
