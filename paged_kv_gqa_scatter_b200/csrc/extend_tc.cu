// Causal extend attention on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
//
// What it computes: "深入解析 mini-sglang" (yunpan.plus), chunked prefill -- a
// chunk of a request attends to the KV its earlier chunks left in the pool,
// reached through the request's page-table row, plus its own rows;
// "Mini-SGLang 完整剖析" (blog.rzhang-lab.cn/post/3) §4.2.3 -- the chunk holds
// extend_len = device_len - cached_len tokens after a cached prefix that may be
// radix-shared (§1.4); §1.2 -- prefill is compute bound.  Query i of a chunk
// sits at position prefix + i and sees keys 0 .. prefix + i; query head h
// reads KV head h / (Hq/Hkv).
//
// Design (B200, one CTA per SM, 11 warps):
//  * A CTA owns one (request, KV head, 2 x 128 query rows) block.  Rows are
//    (token, query head of the group) pairs, token-major, so the G query heads
//    sharing a KV head form the M dimension of one MMA and every K/V tile is
//    used by 256 rows.  The grid is (KV head, query block, request) with the
//    heaviest query block first, and blocks are dispatched in that linear
//    order, so the longest CTAs start first.
//  * warps 8 and 9 -- K/V loads in 64-key steps through a 4-stage ring; warp
//    8 loads the even steps, warp 9 the odd ones.  For each step a warp
//    translates the keys' slots through the page table (one step ahead) and
//    moves the 256-byte head rows with 16-byte cp.async copies straight into
//    the 128-byte-swizzled UMMA operand layout: K-major for K (B of Q K^T),
//    MN-major for V (B of P V).  Two half-warps cover two rows per
//    instruction, so every warp access is two fully used 256-byte segments.
//    (TMA tile::gather4 was tried first: four 128-byte rows per instruction
//    issued too slowly to feed the tensor core.)
//  * warp 10 -- the two Q tiles by 3-D TMA boxes [tokens][G heads][64 dims]
//    (128-byte swizzle), TMEM allocation, and MMA issue: S_i = Q_i K^T into
//    TMEM (M=128, N=64, K=16 steps), then O_i += P_i V (N=128) with P_i read
//    from TMEM.  The whole warp runs the issue loop so descriptors stay
//    warp-uniform; one elected lane issues.  Issue order PV_0(j), QK_0(j+2),
//    PV_1(j), QK_1(j+2): scores are always two steps ahead of the softmax.
//    Completion is signalled with tcgen05.commit to mbarriers.
//  * warps 0-3 and 4-7 -- softmax for Q tile 0 and 1: one thread per row, the
//    step's 64 scores read from TMEM in one go, log2-domain online softmax
//    with a lazily moved max (O rescaled in TMEM only when the max grows by
//    more than 2^8), P written back over S as packed bf16 with tcgen05.st; at
//    the end O / l is read from TMEM and stored as bf16 (prefix mode: O and
//    (max, sum) as fp32 partials).
//  * TMEM (512 columns): S_0 and S_1 as two 64-column halves each (double
//    buffered by step parity), O_0, O_1 128 fp32 columns each; P overwrites
//    the first 32 columns of its S half.
//  * Every mbarrier wait is bounded (about one second); on a timeout the CTA
//    records PKV_DEV_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and
//    returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

constexpr int kRowsPerTile = 128;
constexpr int kKeysPerStep = 64;                  // keys per softmax step / K,V ring stage
constexpr int kQTiles = 2;
constexpr int kKvStages = 4;
constexpr int kQHalfBytes = 128 * 128;            // 128 rows x 64 bf16 (one 128-byte column block)
constexpr int kQTileBytes = 2 * kQHalfBytes;      // 128 rows x 128 bf16
constexpr int kKvHalfBytes = kKeysPerStep * 128;  // 64 keys x 64 bf16
constexpr int kKvTileBytes = 2 * kKvHalfBytes;    // 64 keys x 128 bf16
constexpr int kThreads = 352;  // 11 warps
constexpr int kWarpLoad0 = 8;   // warps 8 and 9: K/V gathers (even / odd steps)
constexpr int kWarpMma = 10;    // MMA issue, Q load, TMEM allocation
constexpr int kLoadThreads = 32;

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kQTileBytes;
constexpr int kOffV = kOffK + kKvStages * kKvTileBytes;
constexpr int kOffBar = kOffV + kKvStages * kKvTileBytes;
constexpr int kNumBars = 32;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack for manual 1024-byte alignment

// Barrier indices.  Barriers touched once per step come in pairs indexed by
// the step's parity (S half), so none can run two phases ahead of its waiter.
constexpr int kBarQFull = 0;
constexpr int kBarKFull = 1;    // + stage (4)
constexpr int kBarKEmpty = 5;   // + stage
constexpr int kBarVFull = 9;    // + stage
constexpr int kBarVEmpty = 13;  // + stage
constexpr int kBarSFull = 17;   // + 2 * q tile + half
constexpr int kBarPReady = 21;  // + 2 * q tile + half
constexpr int kBarODone = 25;   // + q tile
constexpr int kBarOFinal = 27;
constexpr int kBarQReady = 28;  // FP8 pools: Q converted to f16 in place

// TMEM columns: S_i (two 64-column halves, one per step parity) and O_i.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // + 128 * tile + 64 * half
constexpr uint32_t kColO = 256;  // + 128 * tile

constexpr float kRescaleThreshold = 8.0f;

struct ExtendTcArgs {
  const uint8_t* kbase;  // layer base of the K plane (bytes)
  const uint8_t* vbase;
  int64_t slot_stride_bytes;
  const int32_t* table;
  int64_t table_rows, table_cols, table_stride;
  int32_t page_size;
  int64_t num_slots;
  const int32_t* table_idx;
  const int32_t* prefix_lens;
  const int32_t* extend_lens;
  const int32_t* q_offsets;
  int64_t total_q;
  int32_t max_extend;
  __nv_bfloat16* out;
  int32_t hq, hkv;
  float scale_log2;
  int32_t* err;
  // Prefix mode (the shared-prefix pass of cascade decode).  blockIdx.z =
  // group * nsplit + split; q_offsets are the group offsets, prefix_lens the
  // groups' shared prefix lengths.  Every query row of group g (one decode
  // token per member request, no causal mask) attends to keys
  // [split * split_keys, min(p_g, (split + 1) * split_keys)) of the group
  // leader's table row and writes an un-normalised fp32 partial plus its
  // (max, sum) instead of bf16 output.
  int32_t prefix_mode;
  int32_t nsplit, split_keys;
  int32_t nreq;    // query rows (requests) in q
  float2* pre_ml;  // [nsplit][nreq][hq]
  float* pre_o;    // [nsplit][nreq][hq][128]
  float v_scale;   // FP8 pools: V dequantisation scale (1 otherwise)
};

// ---- PTX wrappers -----------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// SMEM matrix descriptor: 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;   // version
  d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
  return d;
}

// Instruction descriptors, kind::f16: bf16 A/B (f16 A/B for FP8 pools, whose
// codes widen exactly to f16), fp32 D, M = 128.
constexpr uint32_t kIdescF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);
constexpr uint32_t kIdescHalf = (1u << 4) | ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescF16 | ((64u >> 3) << 17);                // N = 64 keys, A and B K-major
constexpr uint32_t kIdescPV = kIdescF16 | ((128u >> 3) << 17) | (1u << 16);  // N = 128 dims, B (V) MN-major
constexpr uint32_t kIdescQKHalf = kIdescHalf | ((64u >> 3) << 17);
constexpr uint32_t kIdescPVHalf = kIdescHalf | ((128u >> 3) << 17) | (1u << 16);

// Two floats -> f16x2 (round to nearest even), a in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 16 E4M3 codes -> 16 f16 values (exact), as two 16-byte words.
__device__ __forceinline__ void e4m3x16_to_f16(const uint4& w, uint4& lo, uint4& hi) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] >> 16), __NV_E4M3);
    o[2 * i] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    o[2 * i + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Load 64 consecutive 32-bit TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld64_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
      " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x on the SFU (approximate, flushes subnormal results to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One lane of the (fully active) warp: true in exactly one lane.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ---- the kernel ---------------------------------------------------------------
// kFp8: the pool holds E4M3 codes.  The load warps widen each K/V row to f16
// on the way into shared memory, the softmax warps convert the bf16 Q tiles
// to f16 in place, and the MMAs run on f16 operands (P is packed as f16).
template <int G, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    extend_tc_kernel(const __grid_constant__ CUtensorMap qmap, const ExtendTcArgs a) {
  constexpr uint32_t kIdQK = kFp8 ? kIdescQKHalf : kIdescQK;
  constexpr uint32_t kIdPV = kFp8 ? kIdescPVHalf : kIdescPV;
  constexpr int kRowBytes = kFp8 ? 128 : 256;  // one KV head of one slot in the pool
  constexpr int TQ = kRowsPerTile / G;  // tokens per Q tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + kOffMisc + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int r = a.prefix_mode ? static_cast<int>(blockIdx.z) / a.nsplit : static_cast<int>(blockIdx.z);
  const int split = a.prefix_mode ? static_cast<int>(blockIdx.z) % a.nsplit : 0;
  // Blocks are dispatched in linear order (x fastest): all KV heads of the
  // heaviest query block first, so the whole grid runs longest-first.
  const int qb = static_cast<int>(gridDim.y) - 1 - static_cast<int>(blockIdx.y);

  // ---- block-uniform work description (identical in every thread) ---------
  const int32_t p = a.prefix_lens[r];
  const int64_t qbase = a.q_offsets[r];
  const int32_t e = a.prefix_mode ? static_cast<int32_t>(a.q_offsets[r + 1] - qbase) : a.extend_lens[r];
  if (p < 0 || e < 0 || qbase < 0 || qbase + e > a.total_q) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && g == 0) set_err(a.err, PKV_DEV_ERR_BAD_LENGTH);
    return;
  }
  if (e > a.max_extend && threadIdx.x == 0 && blockIdx.y == 0 && g == 0)
    set_err(a.err, PKV_DEV_ERR_BAD_LENGTH);
  const int i0 = qb * (kQTiles * TQ);
  if (i0 >= e) return;
  // Q tile 1 holds a valid token only if the block has more than TQ of them;
  // otherwise (the last block of a short chunk) its MMAs and softmax are skipped.
  const bool tile1 = i0 + TQ < e;
  // Prefix mode reads the keys through the row of the group's first member.
  const int32_t trow = a.table_idx[a.prefix_mode ? qbase : r];
  const bool row_ok = trow >= 0 && trow < a.table_rows;
  // Keys key0 .. kv_end - 1 are this CTA's (key0 is a multiple of the step).
  const int64_t key0 = a.prefix_mode ? static_cast<int64_t>(split) * a.split_keys : 0;
  int64_t kv_end = a.prefix_mode ? min(static_cast<int64_t>(p), key0 + a.split_keys)
                                 : static_cast<int64_t>(p) + min(e, i0 + kQTiles * TQ);
  if (kv_end > a.table_cols) {
    if (threadIdx.x == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
    kv_end = a.table_cols;
  }
  if (!row_ok && threadIdx.x == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
  if (kv_end <= key0) {
    // Prefix mode only (a causal block always has a key): an empty split
    // leaves an empty partial, (max, sum) = (-inf, 0), which the merge skips.
    if (warp < kWarpLoad0) {
      const int m = (warp & 3) * 32 + lane;
      const int tok = i0 + (warp >> 2) * TQ + m / G;
      if (tok < e)
        a.pre_ml[(static_cast<int64_t>(split) * a.nreq + qbase + tok) * a.hq + g * G + m % G] =
            make_float2(-INFINITY, 0.f);
    }
    return;
  }
  const int nsteps = static_cast<int>((kv_end - key0 + kKeysPerStep - 1) / kKeysPerStep);

  // ---- setup: barriers and TMEM ------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarQFull], 1);
    for (int st = 0; st < kKvStages; ++st) {
      mbar_init(&bars[kBarKFull + st], kLoadThreads);
      mbar_init(&bars[kBarKEmpty + st], 1);
      mbar_init(&bars[kBarVFull + st], kLoadThreads);
      mbar_init(&bars[kBarVEmpty + st], 1);
    }
    for (int b = 0; b < 2 * kQTiles; ++b) {
      mbar_init(&bars[kBarSFull + b], 1);
      mbar_init(&bars[kBarPReady + b], 128);
    }
    for (int i = 0; i < kQTiles; ++i) mbar_init(&bars[kBarODone + i], 1);
    mbar_init(&bars[kBarOFinal], 1);
    mbar_init(&bars[kBarQReady], 2 * 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint8_t* sQ = smem + kOffQ;
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;

  if (warp >= kWarpLoad0 && warp < kWarpMma) {
    // ============================ K/V gathers =================================
    // Warp par loads steps par, par + 2, ... into ring stages (step % 4).  For
    // each 64-key step it translates the keys' slots through the page table
    // (one step ahead) and moves their 256-byte head rows as 16-byte cp.async
    // chunks: in each instruction lanes 0-15 and 16-31 cover the rows of two
    // keys, so a warp access is two fully used 256-byte segments.  Chunk c of
    // key k lands at column block c/8, row k, 16-byte slot (c%8) ^ (k%8): the
    // 128-byte-swizzled UMMA operand layout (K-major for K, MN-major for V).
    // K and V copies of a step are in flight together; the warp waits for
    // each group in turn, makes it visible to the tensor core
    // (fence.proxy.async) and arrives on the stage's full barrier, K first.
    const int par = warp - kWarpLoad0;
    const int h = lane >> 4, c = lane & 15;
    const int32_t* rowp = a.table + (row_ok ? trow : 0) * a.table_stride;
    // A masked key reads the request's first key row (finite, part of its context).
    int32_t dummy = 0;
    if (row_ok) {
      const int64_t s0 = token_slot(rowp, 0, a.page_size, a.num_slots, nullptr);
      dummy = s0 >= 0 ? static_cast<int32_t>(s0) : 0;
    }
    // Slots of keys u*32 + lane (u < 2) of step jj.
    auto lookup = [&](int jj, int32_t (&sl)[2]) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int64_t key = key0 + static_cast<int64_t>(jj) * kKeysPerStep + u * 32 + lane;
        int64_t sv = -1;
        if (jj < nsteps && key < kv_end && row_ok) sv = token_slot(rowp, key, a.page_size, a.num_slots, a.err);
        sl[u] = sv >= 0 ? static_cast<int32_t>(sv) : dummy;
      }
    };
    auto copy_step = [&](const uint8_t* base, uint32_t dst_tile, const int32_t (&sl)[2]) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int kk = u * 32 + 2 * t + h;  // key within the step
          const int32_t slot = __shfl_sync(0xffffffffu, sl[u], 2 * t + h);
          const uint8_t* src = base + static_cast<int64_t>(slot) * a.slot_stride_bytes + g * kRowBytes + c * 16;
          const uint32_t dst = dst_tile + (c >> 3) * kKvHalfBytes + kk * 128 + (((c & 7) ^ (kk & 7)) << 4);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // FP8: 8 lanes per key row (16 codes each, one 16-byte load), 4 rows per
    // instruction; every load of the step is issued before the first
    // conversion, and each 16-code chunk becomes two f16 chunks of the same
    // swizzled layout, stored with plain shared-memory stores.
    auto copy_step_f8 = [&](const uint8_t* base, uint8_t* dst_tile, const int32_t (&sl)[2]) {
      const int q4 = lane >> 3, cf = lane & 7;
#pragma unroll
      for (int u = 0; u < 2; ++u) {  // keys u*32 .. u*32 + 31: 8 loads in flight per lane
        uint4 raw[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int kk = u * 32 + it * 4 + q4;
          const int32_t slot = __shfl_sync(0xffffffffu, sl[u], kk & 31);
          raw[it] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(slot) * a.slot_stride_bytes +
                                                         g * kRowBytes + cf * 16));
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int kk = u * 32 + it * 4 + q4;
          uint4 lo, hi;
          e4m3x16_to_f16(raw[it], lo, hi);
          const int c0 = 2 * cf, c1 = 2 * cf + 1;
          *reinterpret_cast<uint4*>(dst_tile + (c0 >> 3) * kKvHalfBytes + kk * 128 + (((c0 & 7) ^ (kk & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst_tile + (c1 >> 3) * kKvHalfBytes + kk * 128 + (((c1 & 7) ^ (kk & 7)) << 4)) = hi;
        }
      }
    };
    int32_t sl[2];
    lookup(par, sl);
    for (int j = par; j < nsteps; j += 2) {
      const int st = j % kKvStages, use = j / kKvStages;
      if (use >= 1) {
        const bool w = mbar_wait(&bars[kBarKEmpty + st], (use - 1) & 1) &&
                       mbar_wait(&bars[kBarVEmpty + st], (use - 1) & 1);
        if (__any_sync(0xffffffffu, !w || *abort_flag != 0)) {
          if (lane == 0 && !w) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
      int32_t nsl[2];
      if constexpr (kFp8) {
        copy_step_f8(a.kbase, sK + st * kKvTileBytes, sl);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[kBarKFull + st]);
        lookup(j + 2, nsl);
        copy_step_f8(a.vbase, sV + st * kKvTileBytes, sl);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[kBarVFull + st]);
      } else {
        // K and V copies of the step fly together; K is signalled first.
        copy_step(a.kbase, smem_u32(sK + st * kKvTileBytes), sl);
        copy_step(a.vbase, smem_u32(sV + st * kKvTileBytes), sl);
        lookup(j + 2, nsl);  // this warp's next step; the loads fly with the copies
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[kBarKFull + st]);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars[kBarVFull + st]);
      }
      sl[0] = nsl[0];
      sl[1] = nsl[1];
    }
    // No copy into this CTA's shared memory may outlive the loop.
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kWarpMma) {
    // ============================ Q load + MMA issue ==========================
    // Step j writes S_i half (j % 2).  Issue order: QK_0(0), QK_1(0), QK_0(1),
    // QK_1(1), then per step PV_0(j), QK_0(j+2), PV_1(j), QK_1(j+2): the scores
    // for the next step are always computed before the softmax needs them, and
    // QK_i(j+2) reuses the S half that PV_i(j) has just read P from (the
    // tensor pipe executes in issue order).  The whole warp runs this loop so
    // that descriptors and TMEM addresses stay warp-uniform (uniform
    // registers); one elected lane issues each tcgen05 instruction.
    if (elect_one()) {
      mbar_arrive_expect_tx(&bars[kBarQFull], kQTiles * kQTileBytes);
      for (int i = 0; i < kQTiles; ++i)
        for (int hh = 0; hh < 2; ++hh)
          tma_load_3d(sQ + i * kQTileBytes + hh * kQHalfBytes, &qmap, hh * 64, g * G,
                      static_cast<int>(qbase + i0 + i * TQ), &bars[kBarQFull]);
    }
    __syncwarp();
    // Descriptor bases; k-steps add their byte offset / 16 to the start field.
    const uint64_t q_desc = smem_desc(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = smem_desc(smem_u32(sK), 16, 1024);
    const uint64_t v_desc = smem_desc(smem_u32(sV), kKvHalfBytes, 1024);
    auto issue_qk = [&](int i, int j) {
      const uint32_t d = tmem + kColS + 128 * i + 64 * (j & 1);
      const uint64_t ad = q_desc + static_cast<uint64_t>((i * kQTileBytes) >> 4);
      const uint64_t bd = k_desc + static_cast<uint64_t>(((j % kKvStages) * kKvTileBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ao = static_cast<uint64_t>(((kk >> 2) * kQHalfBytes + (kk & 3) * 32) >> 4);
          const uint64_t bo = static_cast<uint64_t>(((kk >> 2) * kKvHalfBytes + (kk & 3) * 32) >> 4);
          mma_ss(d, ad + ao, bd + bo, kIdQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kBarSFull + 2 * i + (j & 1)]);
      }
      __syncwarp();
    };
    auto issue_pv = [&](int i, int j) {
      const uint32_t d = tmem + kColO + 128 * i;
      const uint32_t pa = tmem + kColS + 128 * i + 64 * (j & 1);
      const uint64_t bd = v_desc + static_cast<uint64_t>(((j % kKvStages) * kKvTileBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(d, pa + kk * 8, bd + static_cast<uint64_t>((kk * 2048) >> 4), kIdPV,
                 (j == 0 && kk == 0) ? 0u : 1u);
        mma_commit(&bars[kBarODone + i]);
      }
      __syncwarp();
    };
    auto commit = [&](int bar) {
      if (elect_one()) mma_commit(&bars[bar]);
      __syncwarp();
    };
    auto wait_all = [&](int bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(&bars[bar], parity));
    };
    bool ok = wait_all(kFp8 ? kBarQReady : kBarQFull, 0);
    for (int j = 0; j < 2 && j < nsteps && ok; ++j) {
      ok = wait_all(kBarKFull + j, 0);
      if (!ok) break;
      tc_fence_after();
      issue_qk(0, j);
      if (tile1) issue_qk(1, j);
      commit(kBarKEmpty + j);
    }
    for (int j = 0; j < nsteps && ok; ++j) {
      const int st = j % kKvStages, use = j / kKvStages;
      const bool more = j + 2 < nsteps;
      const int st2 = (j + 2) % kKvStages, use2 = (j + 2) / kKvStages;
      ok = wait_all(kBarVFull + st, use & 1) && wait_all(kBarPReady + 0 + (j & 1), (j >> 1) & 1);
      if (!ok || __any_sync(0xffffffffu, *abort_flag != 0)) break;
      tc_fence_after();
      issue_pv(0, j);
      if (more) {
        ok = wait_all(kBarKFull + st2, use2 & 1);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, j + 2);
      }
      if (tile1) {
        ok = wait_all(kBarPReady + 2 + (j & 1), (j >> 1) & 1);
        if (!ok || __any_sync(0xffffffffu, *abort_flag != 0)) break;
        tc_fence_after();
        issue_pv(1, j);
      }
      commit(kBarVEmpty + st);
      if (more) {
        if (tile1) issue_qk(1, j + 2);
        commit(kBarKEmpty + st2);
      }
    }
    if (!ok) {
      if (lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // Final commit: O complete (or, after an abort, every issued MMA retired).
    commit(kBarOFinal);
    if (!wait_all(kBarOFinal, 0) && lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
  } else if (warp < kWarpLoad0) {
    // ============================ softmax + epilogue ==========================
    const int i = warp >> 2;         // Q tile
    const int wq = warp & 3;         // TMEM lane quadrant
    const int m = wq * 32 + lane;    // row within the tile
    const int tq = m / G, hh = m % G;
    const int tok = i0 + i * TQ + tq;
    const bool valid = tok < e;
    // Keys < lim are visible: causal in extend, the whole split in prefix mode.
    const int64_t lim = a.prefix_mode ? kv_end : (valid ? static_cast<int64_t>(p) + tok + 1 : 1);
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + kColO + 128 * i;
    float m_run = -INFINITY;
    float2 l2 = make_float2(0.f, 0.f);  // running sum of p, even / odd keys
    const float2 sl2 = make_float2(a.scale_log2, a.scale_log2);
    bool ok = true;
    if constexpr (kFp8) {
      // Convert both Q tiles from bf16 to f16 in place (the swizzle permutes
      // whole 16-byte chunks, so each chunk is converted where it lies), make
      // the stores visible to the tensor core, then release the MMA warp.
      const bool wq = mbar_wait(&bars[kBarQFull], 0);
      if (__any_sync(0xffffffffu, !wq)) ok = false;
      uint4* qc = reinterpret_cast<uint4*>(sQ);
      constexpr int kChunks = kQTiles * kQTileBytes / 16;
#pragma unroll 4
      for (int k = threadIdx.x; k < kChunks; k += 2 * 128) {
        const uint4 w = qc[k];
        const float2 f0 = bf16x2_to_f2(w.x), f1 = bf16x2_to_f2(w.y), f2 = bf16x2_to_f2(w.z), f3 = bf16x2_to_f2(w.w);
        qc[k] = make_uint4(pack_f16x2(f0.x, f0.y), pack_f16x2(f1.x, f1.y), pack_f16x2(f2.x, f2.y),
                           pack_f16x2(f3.x, f3.y));
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars[kBarQReady]);
    }
    const int my_steps = (i == 0 || tile1) ? nsteps : 0;  // tile 1 may have no valid row
    for (int j = 0; j < my_steps; ++j) {
      const int hf = j & 1;
      const uint32_t s_addr = tmem + lane_base + kColS + 128 * i + 64 * hf;
      const bool w = mbar_wait(&bars[kBarSFull + 2 * i + hf], (j >> 1) & 1);
      if (__any_sync(0xffffffffu, !w || *abort_flag != 0)) { ok = false; break; }
      tc_fence_after();
      const int64_t kb = key0 + static_cast<int64_t>(j) * kKeysPerStep;
      // Keys kb .. kb + vis - 1 of this step are visible to this row.
      const int64_t vis64 = lim - kb;
      const int32_t vis = vis64 <= 0 ? 0 : (vis64 >= kKeysPerStep ? kKeysPerStep : static_cast<int32_t>(vis64));
      const bool warp_full = __all_sync(0xffffffffu, vis == kKeysPerStep);
      uint32_t sr[64];
      tmem_ld64_nowait(s_addr, sr);
      tmem_wait_ld();
      float mx = -INFINITY;
      if (warp_full) {
#pragma unroll
        for (int u = 0; u < 64; u += 2) mx = max3f(mx, __uint_as_float(sr[u]), __uint_as_float(sr[u + 1]));
      } else {
#pragma unroll
        for (int u = 0; u < 64; ++u) mx = (u < vis) ? fmaxf(mx, __uint_as_float(sr[u])) : mx;
      }
      mx *= a.scale_log2;
      const bool need = mx > m_run + kRescaleThreshold;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds PV of steps < j; wait until the last of them has retired.
        const bool wo = mbar_wait(&bars[kBarODone + i], (j - 1) & 1);
        if (__any_sync(0xffffffffu, !wo)) { ok = false; break; }
        tc_fence_after();
        const float alpha = need ? ex2_approx(m_run - mx) : 1.f;
        l2.x *= alpha;
        l2.y *= alpha;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(o_addr + c * 32, o);
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] *= alpha;
          tmem_st32(o_addr + c * 32, o);
        }
        tmem_wait_st();
      }
      if (need) m_run = mx;
      const float2 negm2 = make_float2(-m_run, -m_run);
      // p = 2^(s * scale * log2e - m), packed to bf16 over the half's first 32 columns.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t w16[16];
        if (warp_full) {
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(sr[32 * c + u]), __uint_as_float(sr[32 * c + u + 1])),
                                        sl2, negm2);
            const float2 pp = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            l2 = __fadd2_rn(l2, pp);
            w16[u >> 1] = kFp8 ? pack_f16x2(pp.x, pp.y) : pack_bf16x2(pp.x, pp.y);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(sr[32 * c + u]), __uint_as_float(sr[32 * c + u + 1])),
                                        sl2, negm2);
            const float p0 = (32 * c + u < vis) ? ex2_approx(t.x) : 0.f;
            const float p1 = (32 * c + u + 1 < vis) ? ex2_approx(t.y) : 0.f;
            l2 = __fadd2_rn(l2, make_float2(p0, p1));
            w16[u >> 1] = kFp8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
          }
        }
        tmem_st16(s_addr + 16 * c, w16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kBarPReady + 2 * i + hf]);
    }
    const float l_run = l2.x + l2.y;
    if (!ok && lane == 0) {
      set_err(a.err, PKV_DEV_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    bool w = mbar_wait(&bars[kBarOFinal], 0);
    w = __all_sync(0xffffffffu, w);
    tc_fence_after();
    if (w && ok && a.prefix_mode) {
      const int64_t row = (static_cast<int64_t>(split) * a.nreq + qbase + tok) * a.hq + g * G + hh;
      float* dst = a.pre_o + row * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(o_addr + c * 32, o);
        if (valid) {
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const float vs = kFp8 ? a.v_scale : 1.f;
            *reinterpret_cast<float4*>(dst + c * 32 + u) =
                make_float4(o[u] * vs, o[u + 1] * vs, o[u + 2] * vs, o[u + 3] * vs);
          }
        }
      }
      if (valid) a.pre_ml[row] = make_float2(m_run, l_run);
    } else if (w && ok) {
      const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * (kFp8 ? a.v_scale : 1.f);
      __nv_bfloat16* dst = a.out + ((qbase + tok) * a.hq + g * G + hh) * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(o_addr + c * 32, o);
        if (valid) {
#pragma unroll
          for (int u = 0; u < 32; u += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(o[u] * inv, o[u + 1] * inv);
            pk.y = pack_bf16x2(o[u + 2] * inv, o[u + 3] * inv);
            pk.z = pack_bf16x2(o[u + 4] * inv, o[u + 5] * inv);
            pk.w = pack_bf16x2(o[u + 6] * inv, o[u + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c * 32 + u) = pk;
          }
        }
      }
    } else if (lane == 0) {
      set_err(a.err, PKV_DEV_ERR_TIMEOUT);
    }
  }

  // ---- teardown: every role is done with TMEM --------------------------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ---- host side ----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_q_map(CUtensorMap* map, const void* q, int32_t hq, int64_t total_q, int G) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(hq), static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(hq) * 128 * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G)};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, bool kFp8>
cudaError_t launch_g(const CUtensorMap& qm, const ExtendTcArgs& a,
                     int64_t grid_z, int32_t max_extend, cudaStream_t s) {
  constexpr int TQ = kRowsPerTile / G;
  const int nqb = (max_extend + kQTiles * TQ - 1) / (kQTiles * TQ);
  static int smem_state[kMaxDevicesHost] = {};
  cudaError_t e = ensure_smem_limit(extend_tc_kernel<G, kFp8>, kSmemBytes, smem_state);
  if (e != cudaSuccess) return e;
  if (grid_z > 65535) return cudaErrorInvalidValue;
  if (nqb > 65535) return cudaErrorInvalidValue;
  dim3 grid(a.hkv, nqb, static_cast<unsigned>(grid_z));
  extend_tc_kernel<G, kFp8><<<grid, kThreads, kSmemBytes, s>>>(qm, a);
  return cudaGetLastError();
}

template <bool kFp8>
cudaError_t launch_any_g(int G, const CUtensorMap& qm, const ExtendTcArgs& a, int64_t grid_z,
                         int32_t max_extend, cudaStream_t s) {
  switch (G) {
    case 1: return launch_g<1, kFp8>(qm, a, grid_z, max_extend, s);
    case 2: return launch_g<2, kFp8>(qm, a, grid_z, max_extend, s);
    case 4: return launch_g<4, kFp8>(qm, a, grid_z, max_extend, s);
    case 8: return launch_g<8, kFp8>(qm, a, grid_z, max_extend, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_for_pool(const PoolView& pool, int G, const CUtensorMap& qm, const ExtendTcArgs& a,
                            int64_t grid_z, int32_t max_extend, cudaStream_t s) {
  return pool.dtype == PKV_DTYPE_FP8_E4M3 ? launch_any_g<true>(G, qm, a, grid_z, max_extend, s)
                                          : launch_any_g<false>(G, qm, a, grid_z, max_extend, s);
}

}  // namespace

cudaError_t launch_extend_tc(const PoolView& pool, const TableView& t, const void* q, int32_t num_q_heads,
                             const int32_t* table_idx, const int32_t* prefix_lens, const int32_t* extend_lens,
                             const int32_t* q_offsets, int32_t batch, int64_t total_q, int32_t max_extend,
                             float scale, void* out, int32_t* err, cudaStream_t s) {
  if (batch == 0 || max_extend == 0 || total_q == 0) return cudaSuccess;
  const int G = num_q_heads / pool.num_kv_heads;
  CUtensorMap qm;
  if (!make_q_map(&qm, q, num_q_heads, total_q, G)) return cudaErrorInvalidValue;
  ExtendTcArgs a;
  a.kbase = pool.k;
  a.vbase = pool.v;
  a.slot_stride_bytes = pool.slot_stride_bytes;
  a.table = t.entries;
  a.table_rows = t.rows;
  a.table_cols = t.cols;
  a.table_stride = t.row_stride;
  a.page_size = pool.page_size;
  a.num_slots = pool.num_slots;
  a.table_idx = table_idx;
  a.prefix_lens = prefix_lens;
  a.extend_lens = extend_lens;
  a.q_offsets = q_offsets;
  a.total_q = total_q;
  a.max_extend = max_extend;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.hq = num_q_heads;
  a.hkv = pool.num_kv_heads;
  a.scale_log2 = scale * kLog2e * pool.k_scale;
  a.err = err;
  a.prefix_mode = 0;
  a.nsplit = 1;
  a.split_keys = 0;
  a.nreq = 0;
  a.pre_ml = nullptr;
  a.pre_o = nullptr;
  a.v_scale = pool.v_scale;
  return launch_for_pool(pool, G, qm, a, batch, max_extend, s);
}

cudaError_t launch_extend_prefix(const PoolView& pool, const TableView& t, const void* q,
                                 int32_t num_q_heads, const int32_t* table_idx,
                                 const int32_t* group_offsets, const int32_t* group_prefix,
                                 int32_t num_groups, int32_t batch, int32_t nsplit, int32_t split_keys,
                                 float scale, float2* pre_ml, float* pre_o, int32_t* err, cudaStream_t s) {
  if (batch == 0 || num_groups == 0 || nsplit == 0) return cudaSuccess;
  if (split_keys % kKeysPerStep != 0) return cudaErrorInvalidValue;
  const int G = num_q_heads / pool.num_kv_heads;
  CUtensorMap qm;
  if (!make_q_map(&qm, q, num_q_heads, batch, G)) return cudaErrorInvalidValue;
  ExtendTcArgs a;
  a.kbase = pool.k;
  a.vbase = pool.v;
  a.slot_stride_bytes = pool.slot_stride_bytes;
  a.table = t.entries;
  a.table_rows = t.rows;
  a.table_cols = t.cols;
  a.table_stride = t.row_stride;
  a.page_size = pool.page_size;
  a.num_slots = pool.num_slots;
  a.table_idx = table_idx;
  a.prefix_lens = group_prefix;
  a.extend_lens = nullptr;
  a.q_offsets = group_offsets;
  a.total_q = batch;
  a.max_extend = batch;
  a.out = nullptr;
  a.hq = num_q_heads;
  a.hkv = pool.num_kv_heads;
  a.scale_log2 = scale * kLog2e * pool.k_scale;
  a.err = err;
  a.prefix_mode = 1;
  a.nsplit = nsplit;
  a.split_keys = split_keys;
  a.nreq = batch;
  a.pre_ml = pre_ml;
  a.pre_o = pre_o;
  a.v_scale = pool.v_scale;
  const int64_t gz = static_cast<int64_t>(num_groups) * nsplit;
  return launch_for_pool(pool, G, qm, a, gz, batch, s);
}

}  // namespace pkv
