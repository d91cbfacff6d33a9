// Fused q/k RMSNorm + RoPE + store_kv: the step between the qkv projection
// and attention, done in one pass over the qkv rows.
//
// What it computes ("Mini-SGLang 完整剖析", blog.rzhang-lab.cn/post/3, §4.6.7):
// the attention layer splits the fused qkv output into q, k and v; Qwen3-style
// models normalise q and k per head (q_norm / k_norm); RoPE rotates q and k in
// place at the batch's positions using the cos/sin cache that one shared
// RotaryEmbedding holds (§4.5.6); the backend then stores k and v into the
// pool at out_loc.  Rotate-half pairing (dims i and i + 64 of a 128-dim head)
// over the whole head; RMSNorm y = x / sqrt(mean(x^2) + eps) * w.
//
// Layout: a half-warp owns one head row of one token (16 lanes x 8 elements):
// the RMS reduction is four xor-shuffles inside the half-warp and the RoPE
// partner of lane c is lane c ^ 8.  Each token has Hq q rows (written to
// q_out), Hkv k rows (written to the pool's K plane) and Hkv v rows (copied to
// the V plane).  All arithmetic is fp32; results round to the pool's type.
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

struct RopeArgs {
  uint8_t* kpool;
  uint8_t* vpool;
  int64_t slot_stride_bytes;
  int64_t num_slots;
  const void* qkv;
  int64_t qkv_row_stride;  // elements
  int32_t hq, hkv;
  const void* positions;
  int32_t pos_i64;
  const float* cos_sin;     // [max_position][128]: 64 cos, then 64 sin
  int64_t max_position;
  const void* q_w;          // [128] or null
  const void* k_w;
  float eps;
  const void* out_loc;
  int32_t loc_i64;
  int64_t n;
  void* q_out;              // [n][hq][128]
  int32_t* err;
};

template <typename E>
__device__ __forceinline__ void load_w8(const void* w, int c, float (&f)[8]) {
  float2 p[4];
  load8<E>(static_cast<const E*>(w) + 8 * c, p);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = p[e].x;
    f[2 * e + 1] = p[e].y;
  }
}

template <typename E>
__global__ void __launch_bounds__(256) qk_norm_rope_store_kernel(const RopeArgs a) {
  const int64_t rows_per_token = a.hq + 2 * a.hkv;
  const int64_t task = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int c = threadIdx.x & 15;  // 8-element chunk of the head row
  const bool active = task < a.n * rows_per_token;
  // The 16 lanes of a half-warp share one task and follow the same path; the
  // two halves of a warp may not (a v row returns early), so every shuffle is
  // restricted to its own half.
  const unsigned hmask = (threadIdx.x & 16) ? 0xffff0000u : 0x0000ffffu;
  const int64_t t = active ? task / rows_per_token : 0;
  const int hr = active ? static_cast<int>(task - t * rows_per_token) : 0;
  const int kind = hr < a.hq ? 0 : (hr < a.hq + a.hkv ? 1 : 2);  // q, k, v
  const int head = kind == 0 ? hr : (kind == 1 ? hr - a.hq : hr - a.hq - a.hkv);
  const E* src = static_cast<const E*>(a.qkv) + t * a.qkv_row_stride + static_cast<int64_t>(hr) * kHeadDim;

  int64_t slot = 0;
  bool slot_ok = true;
  if (kind != 0) {
    slot = a.loc_i64 ? static_cast<const int64_t*>(a.out_loc)[t]
                     : static_cast<int64_t>(static_cast<const int32_t*>(a.out_loc)[t]);
    slot_ok = slot >= 0 && slot < a.num_slots;
    if (!slot_ok && active && c == 0 && kind == 1 && head == 0) set_err(a.err, PKV_DEV_ERR_SLOT_RANGE);
  }

  float2 x2[4];
  if (active) load8<E>(src + 8 * c, x2);
  float x[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = active ? x2[e].x : 0.f;
    x[2 * e + 1] = active ? x2[e].y : 0.f;
  }

  if (kind == 2) {  // v: plain copy (bit exact)
    if (active && slot_ok) {
      E* dst = reinterpret_cast<E*>(a.vpool + slot * a.slot_stride_bytes) + head * kHeadDim + 8 * c;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src + 8 * c);
      if constexpr (sizeof(E) == 4)
        *reinterpret_cast<uint4*>(dst + 4) = *reinterpret_cast<const uint4*>(src + 8 * c + 4);
    }
    return;
  }

  // RMSNorm over the 128 dims of the row (16 lanes).
  const void* w = kind == 0 ? a.q_w : a.k_w;
  if (w != nullptr) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) ss += __shfl_xor_sync(hmask, ss, off);
    const float inv = rsqrtf(ss * (1.0f / kHeadDim) + a.eps);
    float wf[8];
    load_w8<E>(w, c, wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = x[e] * inv * wf[e];
  }

  // RoPE: lanes 0-7 hold dims 0..63 (x1), lanes 8-15 dims 64..127 (x2).
  int64_t pos = 0;
  if (active) {
    pos = a.pos_i64 ? static_cast<const int64_t*>(a.positions)[t]
                    : static_cast<int64_t>(static_cast<const int32_t*>(a.positions)[t]);
  }
  const bool pos_ok = pos >= 0 && pos < a.max_position;
  if (active && !pos_ok && c == 0 && hr == 0) set_err(a.err, PKV_DEV_ERR_POSITION);
  float cs[8], sn[8];
  {
    const float* row = a.cos_sin + (pos_ok ? pos : 0) * kHeadDim;
    const int i0 = 8 * (c & 7);
    const float4 c0 = *reinterpret_cast<const float4*>(row + i0);
    const float4 c1 = *reinterpret_cast<const float4*>(row + i0 + 4);
    const float4 s0 = *reinterpret_cast<const float4*>(row + 64 + i0);
    const float4 s1 = *reinterpret_cast<const float4*>(row + 64 + i0 + 4);
    cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
    cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
    sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
    sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
  }
  float y[8];
  const float sign = (c < 8) ? -1.f : 1.f;  // x1 cos - x2 sin | x2 cos + x1 sin
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float partner = __shfl_xor_sync(hmask, x[e], 8);
    y[e] = pos_ok ? fmaf(sign * partner, sn[e], x[e] * cs[e]) : 0.f;
  }
  if (!active) return;
  if (kind == 0) {
    E* dst = static_cast<E*>(a.q_out) + (t * a.hq + head) * kHeadDim + 8 * c;
    store8<E>(dst, y);
  } else if (slot_ok) {
    E* dst = reinterpret_cast<E*>(a.kpool + slot * a.slot_stride_bytes) + head * kHeadDim + 8 * c;
    store8<E>(dst, y);
  }
}

}  // namespace

cudaError_t launch_qk_norm_rope_store(const PoolView& pool, const void* qkv, int64_t qkv_row_stride,
                                      int32_t num_q_heads, const void* positions, bool pos_i64,
                                      const float* cos_sin, int64_t max_position, const void* q_w,
                                      const void* k_w, float eps, const void* out_loc, bool loc_i64,
                                      int64_t n, void* q_out, int32_t* err, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  RopeArgs a;
  a.kpool = pool.k_mut;
  a.vpool = pool.v_mut;
  a.slot_stride_bytes = pool.slot_stride_bytes;
  a.num_slots = pool.num_slots;
  a.qkv = qkv;
  a.qkv_row_stride = qkv_row_stride;
  a.hq = num_q_heads;
  a.hkv = pool.num_kv_heads;
  a.positions = positions;
  a.pos_i64 = pos_i64 ? 1 : 0;
  a.cos_sin = cos_sin;
  a.max_position = max_position;
  a.q_w = q_w;
  a.k_w = k_w;
  a.eps = eps;
  a.out_loc = out_loc;
  a.loc_i64 = loc_i64 ? 1 : 0;
  a.n = n;
  a.q_out = q_out;
  a.err = err;
  const int64_t tasks = n * (num_q_heads + 2 * pool.num_kv_heads);
  const int64_t blocks = (tasks * 16 + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (pool.dtype == PKV_DTYPE_BF16)
    qk_norm_rope_store_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  else
    qk_norm_rope_store_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
