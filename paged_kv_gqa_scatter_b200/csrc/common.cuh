// Device helpers shared by the pkv kernels (sm_100a).
//
// Everything that waits here is bounded: a wait that has not completed after
// about one second gives up and reports failure to its caller, which records
// PKV_DEV_ERR_TIMEOUT and winds its kernel down.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

constexpr int kHeadDim = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // one second

__device__ __forceinline__ void set_err(int32_t* err, int bits) {
  if (err != nullptr) atomicOr(err, bits);
}

// ---- bf16 <-> f32 --------------------------------------------------------
// A 32-bit word holds two bf16 values: element 2i in the low half, 2i+1 in
// the high half.  Widening is exact.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }

// Round two floats to bf16 (nearest even) and pack them (lo = a, hi = b).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Load 8 consecutive elements as 4 float2 pairs.
template <typename E>
__device__ __forceinline__ void load8(const E* p, float2 (&f)[4]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float2 (&f)[4]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  f[0] = bf16x2_to_f2(w.x);
  f[1] = bf16x2_to_f2(w.y);
  f[2] = bf16x2_to_f2(w.z);
  f[3] = bf16x2_to_f2(w.w);
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float2 (&f)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = make_float2(a.x, a.y);
  f[1] = make_float2(a.z, a.w);
  f[2] = make_float2(b.x, b.y);
  f[3] = make_float2(b.z, b.w);
}

template <>
__device__ __forceinline__ void load8<__nv_fp8_e4m3>(const __nv_fp8_e4m3* p, float2 (&f)[4]) {
  // E4M3 codes widen exactly to half, then to float.
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  const uint32_t u[2] = {w.x, w.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] >> 16), __NV_E4M3);
    f[2 * i] = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    f[2 * i + 1] = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  }
}

// Two floats -> two E4M3 codes (round to nearest even, saturated to +-448),
// a in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// 8 floats times inv_scale (float32 products) -> 8 E4M3 codes.
__device__ __forceinline__ uint2 quant8_e4m3(const float (&f)[8], float inv_scale) {
  uint2 w;
  w.x = pack_e4m3x2(f[0] * inv_scale, f[1] * inv_scale) | (pack_e4m3x2(f[2] * inv_scale, f[3] * inv_scale) << 16);
  w.y = pack_e4m3x2(f[4] * inv_scale, f[5] * inv_scale) | (pack_e4m3x2(f[6] * inv_scale, f[7] * inv_scale) << 16);
  return w;
}

// Store 8 floats as 8 elements (bf16: round to nearest even).
template <typename E>
__device__ __forceinline__ void store8(E* p, const float (&f)[8]);

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 w;
  w.x = pack_bf16x2(f[0], f[1]);
  w.y = pack_bf16x2(f[2], f[3]);
  w.z = pack_bf16x2(f[4], f[5]);
  w.w = pack_bf16x2(f[6], f[7]);
  *reinterpret_cast<uint4*>(p) = w;
}

template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&f)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// ---- shared memory, mbarriers, bulk copies ------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false after ~1 s.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---- page table -----------------------------------------------------------
// Offset of token (or slot) j inside its page of P tokens: a mask when P is a
// power of two, else a 32-bit remainder.  Token positions and table entries are
// 32-bit (the host rejects tables wider than 2^31 columns).
__device__ __forceinline__ int32_t page_offset(int32_t j, int32_t page_size) {
  return (page_size & (page_size - 1)) == 0 ? (j & (page_size - 1)) : (j % page_size);
}

// Slot of token j of the request in table row `row` (row already checked).
// page_size 1: the entry.  page_size P > 1: the entry at column P*(j/P) is the
// page's first slot (page id * P, so page = entry / P) and the slot is
// page*P + j%P, i.e. entry + j%P.  Returns -1 (and sets an error bit) when the
// entry is not page aligned or the slot is out of range.
__device__ __forceinline__ int64_t token_slot(const int32_t* __restrict__ row_ptr, int64_t j64,
                                              int32_t page_size, int64_t num_slots,
                                              int32_t* err) {
  const int32_t j = static_cast<int32_t>(j64);
  int64_t slot;
  if (page_size == 1) {
    slot = row_ptr[j];
  } else {
    const int32_t off = page_offset(j, page_size);
    const int32_t e = row_ptr[j - off];
    if (page_offset(e, page_size) != 0) {
      set_err(err, PKV_DEV_ERR_PAGE_ALIGN);
      return -1;
    }
    slot = static_cast<int64_t>(e) + off;
  }
  if (slot < 0 || slot >= num_slots) {
    set_err(err, PKV_DEV_ERR_SLOT_RANGE);
    return -1;
  }
  return slot;
}

}  // namespace pkv
