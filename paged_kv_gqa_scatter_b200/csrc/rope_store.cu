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
// Layout: a half-warp owns one head row at a time (16 lanes x 8 elements):
// the RMS reduction is four xor-shuffles inside the half-warp and the RoPE
// partner of lane c is lane c ^ 8.  Each token has Hq q rows (written to
// q_out), Hkv k rows (written to the pool's K plane) and Hkv v rows (copied to
// the V plane).  All arithmetic is fp32; results round to the pool's type.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

constexpr int64_t kSmCountHint = 148;  // B200

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
  float k_inv, v_inv;       // FP8 pool: 1 / dequantisation scale
};

// 8 elements as raw 16-byte words (one for bf16, two for fp32), so that a v
// row can be stored back bit for bit, and their values as floats.
template <typename E>
struct Chunk8 {
  uint4 w[sizeof(E) / 2];
};

template <typename E>
__device__ __forceinline__ void load_raw8(const E* p, Chunk8<E>& r) {
#pragma unroll
  for (int i = 0; i < static_cast<int>(sizeof(E) / 2); ++i) r.w[i] = reinterpret_cast<const uint4*>(p)[i];
}

template <typename E>
__device__ __forceinline__ void store_raw8(E* p, const Chunk8<E>& r) {
#pragma unroll
  for (int i = 0; i < static_cast<int>(sizeof(E) / 2); ++i) reinterpret_cast<uint4*>(p)[i] = r.w[i];
}

__device__ __forceinline__ void to_floats(const Chunk8<__nv_bfloat16>& r, float (&x)[8]) {
  const uint32_t u[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = bf16x2_to_f2(u[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

__device__ __forceinline__ void to_floats(const Chunk8<float>& r, float (&x)[8]) {
  const uint4 a = r.w[0], b = r.w[1];
  const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(u[e]);
}

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

// Block (token, row group).  The kThreads / 16 half-warps of a block walk the
// token's head rows kRif at a time (every row load of a group is issued
// before any of them is used), starting at row group blockIdx.y; the
// gridDim.y blocks of a token interleave their groups.  The token's position,
// slot and cos/sin values are loaded once per half-warp, not once per row.
// Large batches use gridDim.y = 1 (one block walks all rows of a token); small
// ones (a decode step) split a token's rows over several blocks so that every
// row load is in flight at once.
// kFp8: the pool holds E4M3 codes; k and v rows are stored as the codes of
// value * (1 / scale) (E is then bf16, the type of qkv and q_out).
template <typename E, int kThreads, int kRif, int kMinBlocks, bool kFp8>
__global__ void __launch_bounds__(kThreads, kMinBlocks) qk_norm_rope_store_kernel(const RopeArgs a) {
  constexpr int kPoolEsize = kFp8 ? 1 : static_cast<int>(sizeof(E));
  constexpr int kHalfWarps = kThreads / 16;
  // An attention kernel launched next may be scheduled now; it waits for
  // this grid before it reads anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t t = blockIdx.x;
  const int rows = a.hq + 2 * a.hkv;
  const int hw = threadIdx.x >> 4;  // half-warp within the block
  constexpr int kGroupRows = kHalfWarps * kRif;
  const int rfirst = hw + static_cast<int>(blockIdx.y) * kGroupRows;  // first row it owns
  const int rstride = kGroupRows * static_cast<int>(gridDim.y);
  const int c = threadIdx.x & 15;   // 8-element chunk of a head row
  // The 16 lanes of a half-warp follow the same path; the two halves of a
  // warp may not (different row kinds), so every shuffle stays in its half.
  const unsigned hmask = (threadIdx.x & 16) ? 0xffff0000u : 0x0000ffffu;
  if (rfirst >= rows) return;  // whole half-warps only

  const int64_t pos = a.pos_i64 ? static_cast<const int64_t*>(a.positions)[t]
                                : static_cast<int64_t>(static_cast<const int32_t*>(a.positions)[t]);
  const int64_t slot = a.loc_i64 ? static_cast<const int64_t*>(a.out_loc)[t]
                                 : static_cast<int64_t>(static_cast<const int32_t*>(a.out_loc)[t]);
  const bool pos_ok = pos >= 0 && pos < a.max_position;
  const bool slot_ok = slot >= 0 && slot < a.num_slots;
  if (threadIdx.x == 0 && blockIdx.y == 0) {
    if (!pos_ok) set_err(a.err, PKV_DEV_ERR_POSITION);
    if (!slot_ok) set_err(a.err, PKV_DEV_ERR_SLOT_RANGE);
  }
  const E* src_row = static_cast<const E*>(a.qkv) + t * a.qkv_row_stride + 8 * c;
  float cs[8], sn[8];
  {
    const float* cr = a.cos_sin + (pos_ok ? pos : 0) * kHeadDim + 8 * (c & 7);
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(cr));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(cr + 4));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(cr + 64));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(cr + 68));
    cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
    cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
    sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
    sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
  }
  const float sign = (c < 8) ? -1.f : 1.f;  // x1 cos - x2 sin | x2 cos + x1 sin

  for (int r0 = rfirst; r0 < rows; r0 += rstride) {
    Chunk8<E> raw[kRif];
#pragma unroll
    for (int u = 0; u < kRif; ++u) {
      const int r = r0 + kHalfWarps * u;
      if (r < rows) load_raw8<E>(src_row + static_cast<int64_t>(r) * kHeadDim, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < kRif; ++u) {
      const int r = r0 + kHalfWarps * u;
      if (r >= rows) break;
      const int kind = r < a.hq ? 0 : (r < a.hq + a.hkv ? 1 : 2);  // q, k, v
      if (kind == 2) {  // v: bit copy into the pool (FP8: its codes)
        if (slot_ok) {
          uint8_t* dst = a.vpool + slot * a.slot_stride_bytes +
                         ((r - a.hq - a.hkv) * kHeadDim + 8 * c) * kPoolEsize;
          if constexpr (kFp8) {
            float xv[8];
            to_floats(raw[u], xv);
            *reinterpret_cast<uint2*>(dst) = quant8_e4m3(xv, a.v_inv);
          } else {
            store_raw8<E>(reinterpret_cast<E*>(dst), raw[u]);
          }
        }
        continue;
      }
      float x[8];
      to_floats(raw[u], x);
      const void* w = kind == 0 ? a.q_w : a.k_w;
      if (w != nullptr) {  // RMSNorm over the row's 128 dims
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) ss += __shfl_xor_sync(hmask, ss, off);
        const float inv = rsqrtf(ss * (1.0f / kHeadDim) + a.eps);
        float wv[8];  // re-read per row (an L1 hit): registers go to rows in flight
        load_w8<E>(w, c, wv);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = x[e] * inv * wv[e];
      }
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // partner dim i +- 64 lives in lane c ^ 8
        const float partner = __shfl_xor_sync(hmask, x[e], 8);
        y[e] = pos_ok ? fmaf(sign * partner, sn[e], x[e] * cs[e]) : 0.f;
      }
      if (kind == 0) {
        store8<E>(static_cast<E*>(a.q_out) + (t * a.hq + r) * kHeadDim + 8 * c, y);
      } else if (slot_ok) {
        uint8_t* dst = a.kpool + slot * a.slot_stride_bytes + ((r - a.hq) * kHeadDim + 8 * c) * kPoolEsize;
        if constexpr (kFp8)
          *reinterpret_cast<uint2*>(dst) = quant8_e4m3(y, a.k_inv);
        else
          store8<E>(reinterpret_cast<E*>(dst), y);
      }
    }
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
  if (n > 0x7fffffffLL) return cudaErrorInvalidValue;
  // 64-thread blocks (4 half-warps, 4 rows in flight each) at 16 blocks per
  // SM: measured best on B200 among 32-512 threads and 2-8 rows in flight
  // (about 96% of copy bandwidth at 32k tokens of Hq 32 / Hkv 8).  Below
  // about four blocks per SM the rows of a token are split over row groups
  // (blockIdx.y), so that a decode step's few tokens put all their row loads
  // in flight in one pass instead of walking them one group after another.
  const int rif = pool.dtype == PKV_DTYPE_F32 ? 2 : 4;
  const int64_t rows = num_q_heads + 2LL * pool.num_kv_heads;
  const int64_t groups = (rows + 4 * rif - 1) / (4 * rif);
  const int64_t want = 4LL * kSmCountHint;
  int64_t ysplit = 1;
  if (n < want) ysplit = std::min<int64_t>(groups, (want + n - 1) / n);
  const dim3 blocks(static_cast<unsigned>(n), static_cast<unsigned>(ysplit));
  a.k_inv = 1.0f / pool.k_scale;
  a.v_inv = 1.0f / pool.v_scale;
  if (pool.dtype == PKV_DTYPE_BF16)
    qk_norm_rope_store_kernel<__nv_bfloat16, 64, 4, 16, false><<<blocks, 64, 0, s>>>(a);
  else if (pool.dtype == PKV_DTYPE_FP8_E4M3)
    qk_norm_rope_store_kernel<__nv_bfloat16, 64, 4, 16, true><<<blocks, 64, 0, s>>>(a);
  else
    qk_norm_rope_store_kernel<float, 64, 2, 16, false><<<blocks, 64, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
