// Split-KV GQA decode attention over the paged pool.
//
// What it computes: "Mini-SGLang 完整剖析" (blog.rzhang-lab.cn/post/3) §1.2 --
// decode runs one query token per request over that request's whole KV
// history and is bound by memory bandwidth; §4.6.4 -- the history is found
// through the token-granular page table, cache_seqlens being the total KV
// length; §4.5.3 -- Hq/Hkv query heads share one KV head.
//
// Design (B200):
//  * The concatenation of all requests' contexts is cut into gridDim.x equal
//    token ranges, one per CTA of a persistent grid (one CTA per SM).  A range
//    may hold the tail of one request, whole requests and the head of another;
//    each (request, CTA) intersection is a "piece".  Equal ranges balance the
//    HBM traffic across SMs exactly, whatever the length mix.
//  * Warps 0..3 are producers (one for fp32 pools), each copying one plane
//    (K or V) of every other token or page group and arming the stage's full
//    barrier for its own bytes: one warp issuing bulk copies tops out near
//    3 G copies/s.  Stages live in a 3-deep shared-memory ring guarded by
//    full/empty mbarriers.  Pools whose page size is a multiple of
//    16 load a stage as page boxes: one tensor copy per plane for every 16
//    table columns (aligned to 16, so inside one page), 16 consecutive slots
//    of all KV heads (32 KB at Hkv 8, bf16), 128B-swizzled.  Other page sizes
//    translate every token's slot and issue one 1-D bulk copy per token row
//    and plane into rows padded by 16 bytes.
//  * The next Hkv warps are consumers, one per KV head.  bf16 and FP8 pools use
//    tensor cores (mma.sync m16n8k16, fp32 accumulate) with the GQA group as
//    the N dimension: S^T = K Q^T over 16-token tiles, then O^T += V^T P^T,
//    fragments read with ldmatrix (transposed for V).  FP8 codes widen
//    exactly to f16.  Softmax runs in the log2 domain with exp2 and a lazily
//    moved running max (the accumulators are rescaled only when the max grows
//    by more than 2^8); p passes to the PV fragments through a small per-warp
//    buffer.  fp32 pools (the check build) keep CUDA-core dot products with a
//    transposing butterfly reduction and packed f32x2 FMAs.
//  * A piece that covers a whole request writes the final output; other
//    pieces write an un-normalised fp32 partial plus (max, sum) to the
//    workspace and decode_combine_kernel merges them.
//  * Cascade suffix pass (cascade.cu): each request starts at its own table
//    column, every piece writes a partial, and the combine kernel also merges
//    the shared-prefix partials.
//  * FP8 (E4M3) pools: 32 tokens per stage; the K scale is folded into the
//    softmax scale and the V scale into the output.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

constexpr int kMaxBatch = 4096;
constexpr int kStages = 3;
constexpr int kMinTokensPerCta = 32;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Per pool element type: tokens per ring stage (a stage holds 2 x T rows of
// Hkv x 128 elements, 64 KB at Hkv 8) and the type of q and out.
template <typename E>
struct DecodeTraits;
template <>
struct DecodeTraits<__nv_bfloat16> {
  static constexpr int kTokensPerStage = 16;
  using IO = __nv_bfloat16;
};
template <>
struct DecodeTraits<float> {
  static constexpr int kTokensPerStage = 8;
  using IO = float;
};
template <>
struct DecodeTraits<__nv_fp8_e4m3> {  // E4M3 codes; q and out stay bf16
  static constexpr int kTokensPerStage = 32;
  using IO = __nv_bfloat16;
};

struct DecodeArgs {
  const uint8_t* kbase;
  const uint8_t* vbase;
  int64_t slot_stride_bytes;
  int64_t num_slots;
  const int32_t* table;
  int64_t table_rows, table_cols, table_stride;
  int32_t page_size;
  const int32_t* table_idx;
  const int32_t* seq_lens;
  int32_t batch;
  const void* q;
  void* out;
  int32_t hq, hkv;
  float scale_log2;   // softmax scale * log2(e) * K dequantisation scale
  float v_scale;      // V dequantisation scale (FP8 pools; 1 otherwise)
  int32_t row_bytes;  // Hkv * 128 * esize
  int32_t* ws_cum;    // [batch + 1]
  int64_t* ws_per;    // [1]
  float2* ws_ml;      // [(grid + batch) * hq]
  float* ws_o;        // [(grid + batch) * hq * 128]
  int32_t* err;
  // Cascade suffix pass: request r reads context columns kv_start[r] ..
  // seq_lens[r] - 1 only, and every piece writes a partial (the combine
  // kernel merges them with the shared-prefix partials).
  const int32_t* kv_start;  // [batch] or null
  int32_t cascade;
};

// Shared memory layout (bytes), identical on host and device.  A stage holds
// T K rows then T V rows, row_stride bytes apart.
struct DecodeSmem {
  int32_t cum_off, psm_off, ring_off, stage_bytes, total;
};

__host__ __device__ inline DecodeSmem decode_smem_layout(int batch, int hkv, int row_stride, int T,
                                                         int psm_per_warp) {
  DecodeSmem L;
  int off = 2 * kStages * 8 + 16;  // full/empty barriers + abort flag
  L.cum_off = off;
  off += 4 * (batch + 1);
  off = (off + 15) & ~15;
  L.psm_off = off;
  off += hkv * psm_per_warp;
  off = (off + 1023) & ~1023;  // page boxes are 128B-swizzled: 1024-byte aligned
  L.ring_off = off;
  L.stage_bytes = 2 * T * row_stride;
  L.total = off + kStages * L.stage_bytes;
  return L;
}

// Tensor-core consumers (bf16 and FP8 pools) read the ring with ldmatrix,
// eight rows of 16 bytes per matrix.  A 16-byte pad after every row (rows are
// a multiple of 128 bytes) puts those eight rows in eight different bank
// groups.
template <typename E>
struct DecodeLayoutTraits {
  static constexpr bool kMma = sizeof(E) != 4;
  static constexpr int kRowPad = kMma ? 16 : 0;
  // p buffer row per head (16-bit entries): a stage's tokens + 8 (the pad
  // spreads the rows' writes and reads over different banks).
  static constexpr int kPStride = DecodeTraits<E>::kTokensPerStage + 8;
  // Producer warps.  One warp issuing one bulk copy per row tops out near 3 G
  // copies/s (measured on B200: 3.1 TB/s at 1 KB rows); four warps, each
  // copying one plane for every other token, reach the HBM bandwidth.
  static constexpr int kProd = kMma ? 4 : 1;
  // bf16 pools pass p to the PV product as two bf16 terms, p = hi + lo (to
  // about 2^-17 relative), in two buffers; f16 (FP8 pools) keeps 11 bits.
  static constexpr bool kSplitP = kMma && sizeof(E) == 2;
  template <int G>
  static constexpr int psm_per_warp() {  // rows for 8 heads per column tile
    return kMma ? 8 * ((G + 7) / 8) * kPStride * 2 * (kSplitP ? 2 : 1) : 4 * DecodeTraits<E>::kTokensPerStage * G;
  }
};

// ---- mma.sync helpers (m16n8k16, fp32 accumulate) -----------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// c += A (16 x 16, row-major fragment) * B (16 x 8, column-major fragment);
// A and B both bf16 (kF16 = false) or both f16.
template <bool kF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (kF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// The two E4M3 codes in the low (lo_f16x2) or high (hi_f16x2) half of w, low
// byte first -> f16x2, exact.
__device__ __forceinline__ uint32_t lo_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(r) : "r"(w));
  return r;
}
__device__ __forceinline__ uint32_t hi_f16x2(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(r) : "r"(w));
  return r;
}

// One page box (16 slots from `slot`, every KV head) of a pool plane into a
// stage: a 4-D map (64 elements, slot, half row, head) for bf16 rows, a 3-D
// map (128 codes, slot, head) for E4M3 rows; see make_page_map.
template <typename E>
__device__ __forceinline__ void tma_page_box(void* dst, const CUtensorMap* map, int32_t slot, uint64_t* bar,
                                             uint64_t policy) {
  if constexpr (sizeof(E) == 1) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(0), "r"(slot), "r"(0), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(0), "r"(slot), "r"(0), "r"(0), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
  }
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Transposing butterfly over groups of D consecutive lanes (D = 8 or 16).  On
// entry every lane holds V partial sums v[0..V); on exit lane d (its index in
// the group) holds the complete sums of values (V/D)*d .. (V/D)*d + V/D - 1
// (V >= D), or of value d >> (log2 D - log2 V) (V < D; lanes sharing a value
// hold the same sum).  Each level halves the values a lane keeps, so the
// reduction costs about one shuffle per complete sum instead of log2 D.
template <int V, int D>
__device__ __forceinline__ void transpose_reduce(float (&v)[V], int d) {
  int n = V;
#pragma unroll
  for (int off = D / 2; off >= 1; off >>= 1) {
    if (n >= 2) {
      const bool upper = (d & off) != 0;
#pragma unroll
      for (int k = 0; k < V / 2; ++k) {
        if (k < n / 2) {
          const float send = upper ? v[k] : v[k + n / 2];
          const float keep = upper ? v[k + n / 2] : v[k];
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x / 2); }

// p values of query heads 0..G-1 for one token, from the warp's p buffer.
template <int G>
__device__ __forceinline__ void load_p(const float* src, float (&p)[G]) {
  if constexpr (G == 1) {
    p[0] = src[0];
  } else if constexpr (G == 2) {
    const float2 x = *reinterpret_cast<const float2*>(src);
    p[0] = x.x;
    p[1] = x.y;
  } else {
#pragma unroll
    for (int k = 0; k < G; k += 4) {
      const float4 x = *reinterpret_cast<const float4*>(src + k);
      p[k] = x.x;
      p[k + 1] = x.y;
      p[k + 2] = x.z;
      p[k + 3] = x.w;
    }
  }
}

// kPaged: the pool's page size is a multiple of 16 and each ring stage is
// loaded as page boxes (one tensor copy per plane per 16 table columns)
// through kmap / vmap; otherwise one bulk copy per token row per plane.
template <typename E, int G, bool kPaged>
__global__ void __launch_bounds__(32 * 12, 1) decode_split_kernel(const DecodeArgs a,
                                                                 const __grid_constant__ CUtensorMap kmap,
                                                                 const __grid_constant__ CUtensorMap vmap) {
  constexpr int T = DecodeTraits<E>::kTokensPerStage;
  // Shape of the CUDA-core consumers (fp32 pools; the tensor-core consumers
  // set their own below).
  constexpr int SUB = (64 / G < T) ? 64 / G : T;  // tokens per softmax sub-step
  constexpr int HALF = SUB / 2;                    // PV: tokens per lane per sub-step
  // Scores: D lanes share a token (each owns 16/D units of 8 dims), TL =
  // 32/D tokens are in flight per warp step, and a lane keeps V = SPL*G
  // partial sums per sub-step.  D = 8 halves the reduction of D = 16; wide
  // groups (G = 8, whose q would not fit in registers) keep D = 16.  A lane's
  // units are dims 8d and 64 + 8d (16-byte loads of bf16 or fp32 rows).
  constexpr int D = G >= 8 ? 16 : 8;
  constexpr int TL = 32 / D;
  constexpr int UPL = 16 / D;                      // 8-element units per lane
  constexpr int SPL = SUB / TL;                    // tokens per lane per sub-step
  constexpr int V = SPL * G;                       // partial sums per lane
  constexpr int NV = V >= D ? V / D : 1;           // complete sums per lane after reduce
  constexpr int LPH = D / G;                       // lanes of a token group holding one head
  constexpr int kLog2D = ilog2c(D);
  constexpr int kLog2V = ilog2c(V);
  constexpr int ESZ = sizeof(E);
  using IO = typename DecodeTraits<E>::IO;
  static_assert(SUB % TL == 0 && NV <= SPL, "decode sub-step shape");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  // Page-box stages need 1024-byte alignment (the host adds 1 KB of slack).
  uint8_t* smem = kPaged ? reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023))
                         : smem_raw;
  // Let the combine kernel be scheduled early; it waits for this grid anyway.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncons = a.hkv;
  using LT = DecodeLayoutTraits<E>;
  static_assert(!kPaged || LT::kMma, "page-box stages feed the tensor-core consumers");
  const int RS = a.row_bytes + (kPaged ? 0 : LT::kRowPad);  // ring row stride
  const DecodeSmem L = decode_smem_layout(a.batch, a.hkv, RS, T, LT::template psm_per_warp<G>());
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(empty + kStages);
  int32_t* cum = reinterpret_cast<int32_t*>(smem + L.cum_off);
  float* psm = reinterpret_cast<float*>(smem + L.psm_off);
  uint8_t* ring = smem + L.ring_off;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], LT::kProd);  // one expect-tx arrival per producer warp
      mbar_init(&empty[s], ncons);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }

  // Every input (lengths, table rows, page table, pool) may come from the
  // preceding kernel on the stream: wait for it before reading any of them.
  // Launch and the barrier set-up above still overlap its tail.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- plan: prefix sums of clamped context lengths -------------------------
  // One warp: each lane sums a contiguous segment of requests, one shuffle
  // scan combines the segments, and each lane writes its segment's prefixes.
  const int B = a.batch;
  const int nthr = blockDim.x;
  if (warp == 0) {
    const int seg = (B + 31) >> 5;
    const int r0 = min(B, lane * seg);
    const int r1 = min(B, r0 + seg);
    int32_t ssum = 0;
    for (int r = r0; r < r1; ++r) {
      int32_t n = a.seq_lens[r];
      if (blockIdx.x == 0) {
        if (n < 1) set_err(a.err, PKV_DEV_ERR_EMPTY_CONTEXT);
        if (n > a.table_cols) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
      }
      n = n < 0 ? 0 : (n > a.table_cols ? static_cast<int32_t>(a.table_cols) : n);
      if (a.kv_start != nullptr) {  // columns before kv_start[r] are not this pass's
        const int32_t st = a.kv_start[r];
        n = st <= 0 ? n : (st >= n ? 0 : n - st);
      }
      cum[r + 1] = n;
      ssum += n;
    }
    int32_t x = ssum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    int32_t run = x - ssum;  // exclusive prefix of this lane's segment
    for (int r = r0; r < r1; ++r) {
      run += cum[r + 1];
      cum[r + 1] = run;
    }
    if (lane == 0) cum[0] = 0;
  }
  __syncthreads();
  const int64_t total = cum[B];
  int64_t per = (total + gridDim.x - 1) / gridDim.x;
  if (per < kMinTokensPerCta) per = kMinTokensPerCta;
  if (blockIdx.x == 0) {
    for (int r = threadIdx.x; r <= B; r += nthr) a.ws_cum[r] = cum[r];
    if (threadIdx.x == 0) a.ws_per[0] = per;
  }
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t hi = min(total, lo + per);
  if (lo >= hi) return;  // idle CTA (no barrier traffic started)
  // First request whose range contains token lo: largest r with cum[r] <= lo.
  int rfirst = 0;
  {
    int l = 0, h = B;  // invariant cum[l] <= lo
    while (h - l > 1) {
      const int m = (l + h) >> 1;
      if (cum[m] <= lo) l = m; else h = m;
    }
    rfirst = l;
  }

  // Producer warp w copies plane w % 2 (K or V) of the tokens (or page groups)
  // whose index is w / 2 modulo kProd / 2; a single producer copies both
  // planes of everything.  Each arms the stage barrier for its own bytes.
  constexpr int kProd = LT::kProd;
  constexpr int kSlices = kProd >= 2 ? kProd / 2 : 1;
  constexpr int kPlanesPerWarp = kProd >= 2 ? 1 : 2;
  const bool copy_k = kProd == 1 || (warp & 1) == 0;
  const bool copy_v = kProd == 1 || (warp & 1) == 1;
  const bool my_slice = (lane % kSlices) == (kProd >= 2 ? warp / 2 : 0);
  if (warp < kProd) {
    if constexpr (kPaged) {
      // ====================== producer (page boxes) ===========================
      // A stage is NG groups of 16 table columns aligned to 16.  Each group
      // lies inside one page (the page size is a multiple of 16), so it is one
      // tensor copy per plane: 16 consecutive slots of every KV head, which
      // lands 128B-swizzled as [head][half][slot][128 B] (bf16) or
      // [head][slot][128 B] (FP8).  Rows of a group outside the piece are
      // loaded too and masked by the consumers.  Lane n < NG owns group n;
      // table entries are loaded two stages ahead.
      constexpr int NG = T / 16;
      const int box_bytes = 16 * a.row_bytes;
      const uint64_t policy = policy_evict_first();
      struct Cursor {
        int r;
        int64_t j0, jb;  // piece tokens [j0, jb) of the pass, relative to col0
        int32_t col0;    // table column of the pass's token 0
        const int32_t* rowp;
        bool row_ok;
      };
      auto piece_start = [&](int rr, Cursor& c) -> bool {
        for (; rr < B && cum[rr] < hi; ++rr) {
          const int64_t ja = max(lo, (int64_t)cum[rr]) - cum[rr];
          const int64_t jb = min(hi, (int64_t)cum[rr + 1]) - cum[rr];
          if (jb > ja) {
            const int32_t trow = a.table_idx[rr];
            c.row_ok = trow >= 0 && trow < a.table_rows;
            if (!c.row_ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
            c.rowp = a.table + (c.row_ok ? trow : 0) * a.table_stride;
            c.col0 = a.kv_start != nullptr ? max(a.kv_start[rr], 0) : 0;
            c.r = rr;
            c.j0 = ja;
            c.jb = jb;
            return true;
          }
        }
        return false;
      };
      // End column (exclusive) of the stage that starts at the cursor.
      auto stage_end = [&](const Cursor& c) -> int64_t {
        const int64_t cs = c.col0 + c.j0;
        return min((int64_t)c.col0 + c.jb, (cs & ~int64_t(15)) + 16 * NG);
      };
      auto advance = [&](Cursor& c) -> bool {
        const int64_t ce = stage_end(c);
        if (ce < (int64_t)c.col0 + c.jb) {
          c.j0 = ce - c.col0;
          return true;
        }
        return piece_start(c.r + 1, c);
      };
      // First table column of this lane's group of the stage at the cursor.
      auto group_col = [&](const Cursor& c) -> int64_t {
        return ((c.col0 + c.j0) & ~int64_t(15)) + 16 * lane;
      };
      // This lane's raw table entry (its group's page's first slot).
      auto lookup = [&](const Cursor& c, bool have) -> int32_t {
        if (!have || lane >= NG || !c.row_ok) return 0;
        const int64_t col = group_col(c);
        if (col >= stage_end(c)) return 0;
        const int32_t c32 = static_cast<int32_t>(col);
        return c.rowp[c32 - page_offset(c32, a.page_size)];
      };
      Cursor c0{}, c1{}, c2{};
      bool h0 = piece_start(rfirst, c0);
      int32_t e0 = lookup(c0, h0);
      c1 = c0;
      bool h1 = h0 && advance(c1);
      int32_t e1 = lookup(c1, h1);
      c2 = c1;
      bool h2 = h1 && advance(c2);
      int last_use[kStages];
#pragma unroll
      for (int i = 0; i < kStages; ++i) last_use[i] = -1;
      for (int64_t s = 0; h0; ++s) {
        const int32_t e2 = lookup(c2, h2);
        const int slot_i = static_cast<int>(s % kStages);
        const int use = static_cast<int>(s / kStages);
        if (use >= 1) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&empty[slot_i], (use - 1) & 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (__any_sync(0xffffffffu, !ok || *abort_flag != 0)) {
            if (!ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
        uint8_t* kst = ring + slot_i * L.stage_bytes;
        uint8_t* vst = kst + NG * box_bytes;
        const int64_t col = group_col(c0);
        const bool in_stage = lane < NG && col < stage_end(c0);
        int32_t slot = -1;
        if (in_stage && c0.row_ok) {
          if (page_offset(e0, a.page_size) != 0) {
            set_err(a.err, PKV_DEV_ERR_PAGE_ALIGN);
          } else {
            const int64_t sl = static_cast<int64_t>(e0) + page_offset(static_cast<int32_t>(col), a.page_size);
            if (sl < 0 || sl >= a.num_slots)
              set_err(a.err, PKV_DEV_ERR_SLOT_RANGE);
            else
              slot = static_cast<int32_t>(sl);
          }
        }
        const bool load = in_stage && slot >= 0 && my_slice;
        if (in_stage && slot < 0 && my_slice) {
          // Bad entry: the group reads as zeros (error already flagged).
          for (int b = 0; b < box_bytes; b += 16) {
            if (copy_k) *reinterpret_cast<uint4*>(kst + lane * box_bytes + b) = make_uint4(0, 0, 0, 0);
            if (copy_v) *reinterpret_cast<uint4*>(vst + lane * box_bytes + b) = make_uint4(0, 0, 0, 0);
          }
          // Later tensor copies (async proxy) may write these bytes again.
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        const unsigned nload = __popc(__ballot_sync(0xffffffffu, load));
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[slot_i], nload * kPlanesPerWarp * box_bytes);
        __syncwarp();
        if (load) {
          if (copy_k) tma_page_box<E>(kst + lane * box_bytes, &kmap, slot, &full[slot_i], policy);
          if (copy_v) tma_page_box<E>(vst + lane * box_bytes, &vmap, slot, &full[slot_i], policy);
        }
        last_use[slot_i] = use;
        c0 = c1;
        h0 = h1;
        e0 = e1;
        c1 = c2;
        h1 = h2;
        e1 = e2;
        if (h2) h2 = advance(c2);
      }
      if (lane == 0) {
        for (int i = 0; i < kStages; ++i)
          if (last_use[i] >= 0 && !mbar_wait(&full[i], last_use[i] & 1))
            set_err(a.err, PKV_DEV_ERR_TIMEOUT);
      }
    } else {
    // =========================== producer ===================================
    // Page-table entries are loaded two stages ahead of the copies that use
    // them, so the dependent table read overlaps the wait for a free stage.
    const uint64_t policy = policy_evict_first();
    struct Cursor {
      int r;
      int64_t j0, jb;  // piece tokens [j0, jb) of the pass, relative to col0
      int32_t col0;    // table column of the pass's token 0
      const int32_t* rowp;
      bool row_ok;
    };
    // First non-empty piece at or after request rr.
    auto piece_start = [&](int rr, Cursor& c) -> bool {
      for (; rr < B && cum[rr] < hi; ++rr) {
        const int64_t ja = max(lo, (int64_t)cum[rr]) - cum[rr];
        const int64_t jb = min(hi, (int64_t)cum[rr + 1]) - cum[rr];
        if (jb > ja) {
          const int32_t trow = a.table_idx[rr];
          c.row_ok = trow >= 0 && trow < a.table_rows;
          if (!c.row_ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TABLE_RANGE);
          c.rowp = a.table + (c.row_ok ? trow : 0) * a.table_stride;
          c.col0 = a.kv_start != nullptr ? max(a.kv_start[rr], 0) : 0;
          c.r = rr;
          c.j0 = ja;
          c.jb = jb;
          return true;
        }
      }
      return false;
    };
    auto advance = [&](Cursor& c) -> bool {
      if (c.j0 + T < c.jb) {
        c.j0 += T;
        return true;
      }
      return piece_start(c.r + 1, c);
    };
    // This lane's raw table entry for a stage (the slot is derived at use).
    auto lookup = [&](const Cursor& c, bool have) -> int32_t {
      const int64_t j = c.j0 + lane;
      if (!have || lane >= T || j >= c.jb || !c.row_ok) return 0;
      const int32_t j32 = c.col0 + static_cast<int32_t>(j);
      return a.page_size == 1 ? c.rowp[j32] : c.rowp[j32 - page_offset(j32, a.page_size)];
    };
    Cursor c0{}, c1{}, c2{};
    bool h0 = piece_start(rfirst, c0);
    int32_t e0 = lookup(c0, h0);
    c1 = c0;
    bool h1 = h0 && advance(c1);
    int32_t e1 = lookup(c1, h1);
    c2 = c1;
    bool h2 = h1 && advance(c2);
    int last_use[kStages];
#pragma unroll
    for (int i = 0; i < kStages; ++i) last_use[i] = -1;
    for (int64_t s = 0; h0; ++s) {
      const int32_t e2 = lookup(c2, h2);
      const int slot_i = static_cast<int>(s % kStages);
      const int use = static_cast<int>(s / kStages);
      if (use >= 1) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[slot_i], (use - 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (__any_sync(0xffffffffu, !ok || *abort_flag != 0)) {
          if (!ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
      uint8_t* kst = ring + slot_i * L.stage_bytes;
      uint8_t* vst = kst + T * RS;
      const int64_t j = c0.j0 + lane;
      const bool in_piece = lane < T && j < c0.jb;
      int64_t slot = -1;
      if (in_piece && c0.row_ok) {
        bool aligned = true;
        if (a.page_size == 1) {
          slot = e0;
        } else if (page_offset(e0, a.page_size) == 0) {
          slot = static_cast<int64_t>(e0) + page_offset(c0.col0 + static_cast<int32_t>(j), a.page_size);
        } else {
          aligned = false;
          set_err(a.err, PKV_DEV_ERR_PAGE_ALIGN);
        }
        if (aligned && (slot < 0 || slot >= a.num_slots)) {
          set_err(a.err, PKV_DEV_ERR_SLOT_RANGE);
          slot = -1;
        }
      }
      const bool load = in_piece && slot >= 0 && my_slice;
      if (in_piece && slot < 0 && my_slice) {
        // Out-of-range entry: the row reads as zeros (error already flagged).
        for (int b = 0; b < a.row_bytes; b += 16) {
          if (copy_k) *reinterpret_cast<uint4*>(kst + lane * RS + b) = make_uint4(0, 0, 0, 0);
          if (copy_v) *reinterpret_cast<uint4*>(vst + lane * RS + b) = make_uint4(0, 0, 0, 0);
        }
        // Later bulk copies (async proxy) may write these bytes again.
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      const unsigned nload = __popc(__ballot_sync(0xffffffffu, load));
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[slot_i], nload * kPlanesPerWarp * a.row_bytes);
      __syncwarp();
      if (load) {
        if (copy_k)
          bulk_g2s(kst + lane * RS, a.kbase + slot * a.slot_stride_bytes, a.row_bytes, &full[slot_i], policy);
        if (copy_v)
          bulk_g2s(vst + lane * RS, a.vbase + slot * a.slot_stride_bytes, a.row_bytes, &full[slot_i], policy);
      }
      last_use[slot_i] = use;
      // Shift the look-ahead window.
      c0 = c1;
      h0 = h1;
      e0 = e1;
      c1 = c2;
      h1 = h2;
      e1 = e2;
      if (h2) h2 = advance(c2);
    }
    // Make sure no copy into this CTA's shared memory is still in flight.
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i)
        if (last_use[i] >= 0 && !mbar_wait(&full[i], last_use[i] & 1))
          set_err(a.err, PKV_DEV_ERR_TIMEOUT);
    }
    }
    return;
  }

  if constexpr (LT::kMma) {
    // ======================= consumers (tensor cores) =========================
    // Per 16-token tile, with the GQA group as the N dimension (one column
    // tile of 8 heads, two at G = 16):
    //   S^T (16 tokens x 8 heads)  = K (16 x 128) . Q^T (128 x 8)  8 MMAs
    //   O^T (128 dims x 8 heads)  += V^T (128 x 16) . P^T (16 x 8)  8 MMAs
    // Lane (qr, kq) = (lane / 4, lane % 4) holds scores of tokens qr, qr + 8
    // and output columns for heads 2kq, 2kq + 1 of each column tile (columns
    // >= G are padding),
    // so its softmax state (max, sum) covers exactly the heads whose output it
    // accumulates.  P passes from the score layout to the PV B fragment
    // through the warp's p buffer [head][token] (16-bit).  bf16 pools run bf16
    // MMAs on the stored rows, with p as two bf16 terms (hi + lo, two PV MMAs
    // on the same V fragments) so that it keeps about 16 significant bits;
    // FP8 pools widen codes exactly to f16 and run f16 MMAs with p in f16 (q
    // enters as f16 scaled by 2^-8, undone in the score scale).
    constexpr bool kF8 = sizeof(E) == 1;
    constexpr int NT = T / 16;  // 16-token tiles per stage (bf16 1, FP8 2)
    constexpr int kPS = LT::kPStride;
    static_assert(T == 16 * NT, "decode tensor-core stage");
    constexpr float kQPre = kF8 ? 1.f / 256.f : 1.f;
    const int g = warp - kProd;  // KV head
    if (g >= ncons) return;
    const int qr = lane >> 2, kq = lane & 3;
    // The group's heads form NH column tiles of 8 (NH = 2 at G = 16); in tile
    // h this lane's columns are heads 8h + 2kq and 8h + 2kq + 1.
    constexpr int NH = (G + 7) / 8;
    auto hv = [&](int h, int hs) { return 8 * h + 2 * kq + hs < G; };
    const float sl = kF8 ? a.scale_log2 * 256.f : a.scale_log2;
    constexpr bool kSplitP = LT::kSplitP;
    uint16_t* pw = reinterpret_cast<uint16_t*>(smem + L.psm_off) + g * (8 * NH * kPS) * (kSplitP ? 2 : 1);
    uint16_t* pw_lo = pw + 8 * NH * kPS;  // low bf16 terms (bf16 pools)
    const uint32_t ring_s = smem_u32(ring);
    // ldmatrix row of this lane: K (plain) matrices are (tokens 0-7 | 8-15) x
    // (first | second 16 bytes); V (transposed) matrices are (first | second
    // 16 bytes) x (tokens 0-7 | 8-15).
    const int tok_k = (lane & 7) + ((lane >> 3) & 1) * 8, col_k = lane >> 4;
    const int tok_v = (lane & 7) + (lane >> 4) * 8, col_v = (lane >> 3) & 1;
    const int x7 = lane & 7;
    const int box_bytes = 16 * a.row_bytes;  // one page box: 16 slots of all KV heads
    const IO* qbase = static_cast<const IO*>(a.q);
    IO* obase = static_cast<IO*>(a.out);
    int64_t s = 0;
    for (int r = rfirst; r < B && cum[r] < hi; ++r) {
      const int64_t ja = max(lo, (int64_t)cum[r]) - cum[r];
      const int64_t jb = min(hi, (int64_t)cum[r + 1]) - cum[r];
      if (jb <= ja) continue;
      const bool whole = !a.cascade && cum[r] >= lo && cum[r + 1] <= hi;
      if (r + 1 < B && cum[r + 1] < hi && lane < 2 * G)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(qbase + ((int64_t)(r + 1) * a.hq + g * G) * kHeadDim +
                                                        lane * (128 / static_cast<int>(sizeof(IO)))));
      // Q^T B fragments, 16 dims per MMA: b0 = dims k, k + 1 and b1 = dims
      // k + 8, k + 9 (k = 2 kq) of head qr.  FP8 rows use the dim order of
      // their K fragments instead: b0 = dims 4kq, 4kq + 1, b1 = 4kq + 2, 4kq + 3.
      uint32_t qb[NH][8][2];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (8 * h + qr < G) {
          const IO* qrow = qbase + ((int64_t)r * a.hq + g * G + 8 * h + qr) * kHeadDim;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if constexpr (kF8) {
              const uint2 w = *reinterpret_cast<const uint2*>(qrow + 16 * c + 4 * kq);
              qb[h][c][0] = pack_f16x2(bf16_lo(w.x) * kQPre, bf16_hi(w.x) * kQPre);
              qb[h][c][1] = pack_f16x2(bf16_lo(w.y) * kQPre, bf16_hi(w.y) * kQPre);
            } else {
              qb[h][c][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * c + 2 * kq);
              qb[h][c][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * c + 2 * kq + 8);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) qb[h][c][0] = qb[h][c][1] = 0u;
        }
      }
      float acc[8][NH][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][h][e] = 0.f;
      float lsum[NH][2], mrun[NH][2];  // per column head: this lane's share of the sum of p; running max (log2)
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          lsum[h][hs] = 0.f;
          mrun[h][hs] = -INFINITY;
        }

      // Stages: T tokens each (row copies), or NT groups of 16 table columns
      // aligned to 16 (page boxes; a piece's first and last groups may be
      // partial).  Tile nt of a stage holds its valid tokens at box rows
      // [lo_t[nt], hi_t[nt]).
      const int32_t col0 = (kPaged && a.kv_start != nullptr) ? max(a.kv_start[r], 0) : 0;
      int64_t j0 = ja;
      while (j0 < jb) {
        const int slot_i = static_cast<int>(s % kStages);
        const int use = static_cast<int>(s / kStages);
        bool ok = mbar_wait(&full[slot_i], use & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || *abort_flag) {
          if (!ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          return;
        }
        int lo_t[NT], hi_t[NT];
        int64_t jn;
        if constexpr (kPaged) {
          const int64_t cs = col0 + j0, b0 = cs & ~int64_t(15);
          const int64_t ce = min((int64_t)col0 + jb, b0 + 16 * NT);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            lo_t[nt] = static_cast<int>(max(cs - (b0 + 16 * nt), (int64_t)0));
            hi_t[nt] = static_cast<int>(min(ce - (b0 + 16 * nt), (int64_t)16));
          }
          jn = ce - col0;
        } else {
          const int ntok = static_cast<int>(min((int64_t)T, jb - j0));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            lo_t[nt] = 0;
            hi_t[nt] = min(16, ntok - 16 * nt);
          }
          jn = j0 + T;
        }
        const uint32_t kst = ring_s + slot_i * L.stage_bytes;
        const uint32_t vst = kst + T * RS;  // T * row_bytes in page-box stages
        // ldmatrix row addresses of 16-dim chunk c (bf16) or 16-code chunk
        // pair cp (FP8) of tile nt: padded rows, or 128B-swizzled page boxes
        // [head][half (bf16)][16 slots][128 B] (16-byte chunk x of box row t
        // stored at chunk x ^ (t & 7); here t & 7 = lane & 7).
        auto k_addr = [&](int nt, int c) -> uint32_t {
          if constexpr (kPaged) {
            if constexpr (kF8)
              return kst + nt * box_bytes + (g * 16 + tok_k) * 128 + (((2 * c + col_k) ^ x7) << 4);
            else
              return kst + nt * box_bytes + ((g * 2 + (c >> 2)) * 16 + tok_k) * 128 +
                     ((((2 * c + col_k) & 7) ^ x7) << 4);
          } else {
            if constexpr (kF8)
              return kst + (16 * nt + tok_k) * RS + g * kHeadDim + 16 * (2 * c + col_k);
            else
              return kst + (16 * nt + tok_k) * RS + (g * kHeadDim + 16 * c + 8 * col_k) * 2;
          }
        };
        auto v_addr = [&](int nt, int c) -> uint32_t {
          if constexpr (kPaged) {
            if constexpr (kF8)
              return vst + nt * box_bytes + (g * 16 + tok_v) * 128 + (((2 * c + col_v) ^ x7) << 4);
            else
              return vst + nt * box_bytes + ((g * 2 + (c >> 2)) * 16 + tok_v) * 128 +
                     ((((2 * c + col_v) & 7) ^ x7) << 4);
          } else {
            if constexpr (kF8)
              return vst + (16 * nt + tok_v) * RS + g * kHeadDim + 16 * (2 * c + col_v);
            else
              return vst + (16 * nt + tok_v) * RS + (g * kHeadDim + 16 * c + 8 * col_v) * 2;
          }
        };
        // ---- scores: NT independent 16-token tiles, each with two
        // accumulators (even and odd 16-dim chunks) to halve the MMA chain.
        float sc[NT][NH][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float se[NH][4], so[NH][4];
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) se[h][e] = so[h][e] = 0.f;
          if (hi_t[nt] > lo_t[nt]) {
            if constexpr (kF8) {
#pragma unroll
              for (int cp = 0; cp < 4; ++cp) {
                uint32_t w[4];
                ldsm_x4(k_addr(nt, cp), w);
                // w[0], w[1]: tokens 0-7, 8-15 of 16-dim chunk 2cp; w[2], w[3]: chunk 2cp + 1.
                const uint32_t f0[4] = {lo_f16x2(w[0]), lo_f16x2(w[1]), hi_f16x2(w[0]), hi_f16x2(w[1])};
                const uint32_t f1[4] = {lo_f16x2(w[2]), lo_f16x2(w[3]), hi_f16x2(w[2]), hi_f16x2(w[3])};
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                  mma16816<true>(se[h], f0, qb[h][2 * cp][0], qb[h][2 * cp][1]);
                  mma16816<true>(so[h], f1, qb[h][2 * cp + 1][0], qb[h][2 * cp + 1][1]);
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < 8; c += 2) {
                uint32_t f0[4], f1[4];
                ldsm_x4(k_addr(nt, c), f0);
                ldsm_x4(k_addr(nt, c + 1), f1);
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                  mma16816<false>(se[h], f0, qb[h][c][0], qb[h][c][1]);
                  mma16816<false>(so[h], f1, qb[h][c + 1][0], qb[h][c + 1][1]);
                }
              }
            }
          }
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][h][e] = se[h][e] + so[h][e];
        }
        // sc[nt][h] = S[token qr][head 8h + 2kq], S[qr][8h + 2kq + 1],
        // S[qr + 8][8h + 2kq], S[qr + 8][8h + 2kq + 1] of tile nt; scaled to
        // the log2 domain, masked.
        float sv[NT][NH][4];
        float mx[NH][2];
#pragma unroll
        for (int h = 0; h < NH; ++h) mx[h][0] = mx[h][1] = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const bool t0 = qr >= lo_t[nt] && qr < hi_t[nt];
          const bool t1 = qr + 8 >= lo_t[nt] && qr + 8 < hi_t[nt];
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            sv[nt][h][0] = (hv(h, 0) && t0) ? sc[nt][h][0] * sl : -INFINITY;
            sv[nt][h][1] = (hv(h, 1) && t0) ? sc[nt][h][1] * sl : -INFINITY;
            sv[nt][h][2] = (hv(h, 0) && t1) ? sc[nt][h][2] * sl : -INFINITY;
            sv[nt][h][3] = (hv(h, 1) && t1) ? sc[nt][h][3] * sl : -INFINITY;
            mx[h][0] = fmaxf(mx[h][0], fmaxf(sv[nt][h][0], sv[nt][h][2]));
            mx[h][1] = fmaxf(mx[h][1], fmaxf(sv[nt][h][1], sv[nt][h][3]));
          }
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) mx[h][hs] = fmaxf(mx[h][hs], __shfl_xor_sync(0xffffffffu, mx[h][hs], off));
        // Lazy rescale: the max moves only when it grows by more than the
        // threshold (p stays below 2^threshold, well inside f16 and bf16).
        float al[NH][2];
        bool need_any = false;
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
            al[h][hs] = 1.f;
            if (mx[h][hs] > mrun[h][hs] + kRescaleThreshold) {
              al[h][hs] = exp2f(mrun[h][hs] - mx[h][hs]);
              mrun[h][hs] = mx[h][hs];
              lsum[h][hs] *= al[h][hs];
              need_any = true;
            }
          }
        if (__any_sync(0xffffffffu, need_any)) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              acc[mt][h][0] *= al[h][0];
              acc[mt][h][2] *= al[h][0];
              acc[mt][h][1] *= al[h][1];
              acc[mt][h][3] *= al[h][1];
            }
        }
        // p into the buffers [head][token]: f16 (FP8 pools), or bf16 hi and
        // lo terms.
        auto put = [&](int i, float x) {
          if constexpr (kF8) {
            pw[i] = __half_as_ushort(__float2half_rn(x));
          } else {
            const __nv_bfloat16 hb = __float2bfloat16_rn(x);
            pw[i] = __bfloat16_as_ushort(hb);
            if constexpr (kSplitP) pw_lo[i] = __bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(hb)));
          }
        };
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
              if (!hv(h, hs)) continue;
              const float p0 = exp2f(sv[nt][h][hs] - mrun[h][hs]);
              const float p1 = exp2f(sv[nt][h][hs + 2] - mrun[h][hs]);
              lsum[h][hs] += p0 + p1;
              const int row = (8 * h + 2 * kq + hs) * kPS + 16 * nt;
              put(row + qr, p0);
              put(row + qr + 8, p1);
            }
        __syncwarp();
        // P^T B fragments of column tile h: b0 = p of head 8h + qr at tokens
        // 2kq, 2kq + 1 of the tile; b1 at + 8 (pl: the low terms).
        uint32_t pb[NT][NH][2], pl[NT][NH][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            pb[nt][h][0] = pb[nt][h][1] = pl[nt][h][0] = pl[nt][h][1] = 0u;
            if (8 * h + qr < G) {
              const int row = (8 * h + qr) * kPS + 16 * nt + 2 * kq;
              pb[nt][h][0] = *reinterpret_cast<const uint32_t*>(pw + row);
              pb[nt][h][1] = *reinterpret_cast<const uint32_t*>(pw + row + 8);
              if constexpr (kSplitP) {
                pl[nt][h][0] = *reinterpret_cast<const uint32_t*>(pw_lo + row);
                pl[nt][h][1] = *reinterpret_cast<const uint32_t*>(pw_lo + row + 8);
              }
            }
          }
        __syncwarp();
        // ---- PV -------------------------------------------------------------
        // In a partial tile, tokens outside [lo, hi) are not this piece's
        // (stale, unwritten or other pages' rows): their V entries are zeroed
        // in the A fragments, since p = 0 would not clear a non-finite value.
        auto pv_tile = [&](int nt, auto masked_tag) {
          constexpr bool kMasked = decltype(masked_tag)::value;
          uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
          if constexpr (kMasked) {
            const int lo = lo_t[nt], hi = hi_t[nt];
            auto in = [&](int t) { return t >= lo && t < hi; };
            mlo = (in(2 * kq) ? 0x0000ffffu : 0u) | (in(2 * kq + 1) ? 0xffff0000u : 0u);
            mhi = (in(2 * kq + 8) ? 0x0000ffffu : 0u) | (in(2 * kq + 9) ? 0xffff0000u : 0u);
          }
          if constexpr (kF8) {
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              uint32_t w[4];
              ldsm_x4_trans(v_addr(nt, pp), w);
              // w[j] = codes (token 2kq: dims 2qr, 2qr + 1 | token 2kq + 1:
              // same dims) of matrix j = (chunk 2pp | 2pp + 1) x (tokens 0-7 | 8-15).
              uint32_t fe[4], fo[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t x = __byte_perm(w[j], 0u, 0x3120);  // (t0 even, t1 even, t0 odd, t1 odd)
                fe[j] = lo_f16x2(x);
                fo[j] = hi_f16x2(x);
                if constexpr (kMasked) {
                  fe[j] &= j < 2 ? mlo : mhi;
                  fo[j] &= j < 2 ? mlo : mhi;
                }
              }
#pragma unroll
              for (int h = 0; h < NH; ++h) {
                mma16816<true>(acc[2 * pp][h], fe, pb[nt][h][0], pb[nt][h][1]);
                mma16816<true>(acc[2 * pp + 1][h], fo, pb[nt][h][0], pb[nt][h][1]);
              }
            }
          } else {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
              uint32_t f[4];
              ldsm_x4_trans(v_addr(nt, mt), f);
              if constexpr (kMasked) {
                f[0] &= mlo;
                f[1] &= mlo;
                f[2] &= mhi;
                f[3] &= mhi;
              }
#pragma unroll
              for (int h = 0; h < NH; ++h) {
                mma16816<false>(acc[mt][h], f, pb[nt][h][0], pb[nt][h][1]);
                if constexpr (kSplitP) mma16816<false>(acc[mt][h], f, pl[nt][h][0], pl[nt][h][1]);
              }
            }
          }
        };
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (lo_t[nt] == 0 && hi_t[nt] == 16)
            pv_tile(nt, std::false_type{});
          else if (hi_t[nt] > lo_t[nt])
            pv_tile(nt, std::true_type{});
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot_i]);
        j0 = jn;
        ++s;
      }

      // ---- finish the piece -------------------------------------------------
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) lsum[h][hs] += __shfl_xor_sync(0xffffffffu, lsum[h][hs], off);
      // Output dims of accumulator (mt, e): bf16 rows: 16 mt + qr (+ 8 for
      // e >= 2); FP8 rows: 32 (mt / 2) + 2 qr + (mt & 1) (+ 16 for e >= 2).
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          if (!hv(h, hs)) continue;
          const int head = g * G + 8 * h + 2 * kq + hs;
          const float ls = lsum[h][hs], mh = mrun[h][hs];
          const float vs = kF8 ? a.v_scale : 1.f;
          if (whole) {
            const float inv = ls > 0.f ? vs / ls : 0.f;
            IO* orow = obase + ((int64_t)r * a.hq + head) * kHeadDim;
            if constexpr (kF8) {
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) {
#pragma unroll
                for (int up = 0; up < 2; ++up) {
                  const uint32_t w =
                      pack_bf16x2(acc[2 * pp][h][hs + 2 * up] * inv, acc[2 * pp + 1][h][hs + 2 * up] * inv);
                  *reinterpret_cast<uint32_t*>(orow + 32 * pp + 16 * up + 2 * qr) = w;
                }
              }
            } else {
#pragma unroll
              for (int mt = 0; mt < 8; ++mt) {
                orow[16 * mt + qr] = __float2bfloat16_rn(acc[mt][h][hs] * inv);
                orow[16 * mt + qr + 8] = __float2bfloat16_rn(acc[mt][h][hs + 2] * inv);
              }
            }
          } else {
            const int64_t id = static_cast<int64_t>(blockIdx.x) + r;
            float* op = a.ws_o + (id * a.hq + head) * kHeadDim;
            if constexpr (kF8) {
#pragma unroll
              for (int pp = 0; pp < 4; ++pp)
#pragma unroll
                for (int up = 0; up < 2; ++up)
                  *reinterpret_cast<float2*>(op + 32 * pp + 16 * up + 2 * qr) =
                      make_float2(acc[2 * pp][h][hs + 2 * up] * vs, acc[2 * pp + 1][h][hs + 2 * up] * vs);
            } else {
#pragma unroll
              for (int mt = 0; mt < 8; ++mt) {
                op[16 * mt + qr] = acc[mt][h][hs];
                op[16 * mt + qr + 8] = acc[mt][h][hs + 2];
              }
            }
            if (qr == 0) a.ws_ml[id * a.hq + head] = make_float2(mh, ls);
          }
        }
    }
  } else {
  // ===================== consumers (CUDA cores, fp32 pools) ===================
  // Scores use the token-group lane map (tl, d) = (lane / D, lane % D); the
  // PV product uses (half, c) = (lane / 16, lane % 16): lane c owns dims
  // 8c .. 8c+7 and half picks even or odd tokens.  The p values pass from the
  // first map to the second through the warp's p buffer [SUB][G].
  const int g = warp - kProd;  // KV head
  if (g >= ncons) return;
  const int c = lane & 15, half = lane >> 4;
  const int tl = lane / D, d = lane % D;
  // Head and value index of the complete scores this lane holds after the
  // reduction; for V < D, lanes sharing a value let only the first add it
  // to the running sum.
  const int idx0 = V >= D ? NV * d : (d >> (kLog2D - kLog2V));
  const int hl = idx0 / SPL;
  const bool owner = V >= D || (d & ((D >> kLog2V) - 1)) == 0;
  // A lane holding scores of head hh (used to broadcast per-head values).
  auto head_lane = [](int hh) { return hh * LPH; };
  float* pw = psm + g * SUB * G;  // this warp's p buffer [SUB][G]
  // First dim of this lane's score unit m.
  auto unit_dim = [&](int m) { return 8 * (d + D * m); };
  const IO* qbase = static_cast<const IO*>(a.q);
  IO* obase = static_cast<IO*>(a.out);
  int64_t s = 0;
  for (int r = rfirst; r < B && cum[r] < hi; ++r) {
    const int64_t ja = max(lo, (int64_t)cum[r]) - cum[r];
    const int64_t jb = min(hi, (int64_t)cum[r + 1]) - cum[r];
    if (jb <= ja) continue;
    const bool whole = !a.cascade && cum[r] >= lo && cum[r + 1] <= hi;
    // Warm L2 with the next request's queries while this piece runs.
    if (r + 1 < B && cum[r + 1] < hi && lane < 2 * G)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(qbase + ((int64_t)(r + 1) * a.hq + g * G) * kHeadDim +
                                                      lane * (128 / static_cast<int>(sizeof(IO)))));

    // q of this lane's units (pre-scaled by scale * log2 e).
    float2 q2[G][UPL][4];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
#pragma unroll
      for (int m = 0; m < UPL; ++m) {
        load8<IO>(qbase + ((int64_t)r * a.hq + g * G + hh) * kHeadDim + unit_dim(m), q2[hh][m]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          q2[hh][m][e].x *= a.scale_log2;
          q2[hh][m][e].y *= a.scale_log2;
        }
      }
    }
    float2 o2[G][4];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < 4; ++e) o2[hh][e] = make_float2(0.f, 0.f);
    float l_lane = 0.f;       // this lane's share of the sum of p for head hl
    float m_run = -INFINITY;  // running max of head hl (log2 domain)

    for (int64_t j0 = ja; j0 < jb; j0 += T, ++s) {
      const int slot_i = static_cast<int>(s % kStages);
      const int use = static_cast<int>(s / kStages);
      bool ok = mbar_wait(&full[slot_i], use & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok || *abort_flag) {
        if (!ok && lane == 0) set_err(a.err, PKV_DEV_ERR_TIMEOUT);
        *abort_flag = 1;
        return;
      }
      const int ntok = static_cast<int>(min((int64_t)T, jb - j0));
      const uint8_t* kst = ring + slot_i * L.stage_bytes;
      const uint8_t* vst = kst + T * RS;

#pragma unroll
      for (int sub = 0; sub < T; sub += SUB) {
        if (sub >= ntok) break;
        // ---- scores: partial dot products over this lane's units -----------
        float v[V];
#pragma unroll
        for (int i = 0; i < SPL; ++i) {
          const int t = sub + TL * i + tl;
          float2 acc[G];
          float2 kw[UPL][4];
#pragma unroll
          for (int m = 0; m < UPL; ++m)
            load8<E>(reinterpret_cast<const E*>(kst + t * RS + (g * kHeadDim + unit_dim(m)) * ESZ), kw[m]);
#pragma unroll
          for (int m = 0; m < UPL; ++m) {
            const float2 (&k2)[4] = kw[m];
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
              acc[hh] = m == 0 ? __fmul2_rn(k2[0], q2[hh][m][0]) : __ffma2_rn(k2[0], q2[hh][m][0], acc[hh]);
              acc[hh] = __ffma2_rn(k2[1], q2[hh][m][1], acc[hh]);
              acc[hh] = __ffma2_rn(k2[2], q2[hh][m][2], acc[hh]);
              acc[hh] = __ffma2_rn(k2[3], q2[hh][m][3], acc[hh]);
            }
          }
#pragma unroll
          for (int hh = 0; hh < G; ++hh) v[hh * SPL + i] = acc[hh].x + acc[hh].y;
        }
        transpose_reduce<V, D>(v, d);
        // This lane now holds NV complete scores of head hl.
        float sc[NV];
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int tt = TL * ((idx0 + k) % SPL) + tl;
          sc[k] = (sub + tt < ntok) ? v[k] : -INFINITY;
          mx = fmaxf(mx, sc[k]);
        }
#pragma unroll
        for (int off = 1; off < LPH; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
        for (int off = D; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const bool need = mx > m_run + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = exp2f(m_run - mx);
          m_run = mx;
          l_lane *= alpha;
        }
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int tt = TL * ((idx0 + k) % SPL) + tl;
          const float p = exp2f(sc[k] - m_run);
          if (owner) {
            pw[tt * G + hl] = p;
            l_lane += p;
          }
        }
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float al = __shfl_sync(0xffffffffu, alpha, head_lane(hh));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o2[hh][e].x *= al;
              o2[hh][e].y *= al;
            }
          }
        }
        __syncwarp();
        // ---- PV ------------------------------------------------------------
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const int tt = 2 * i + half;
          if (sub + tt < ntok) {
            float2 v2[4];
            load8<E>(reinterpret_cast<const E*>(vst + (sub + tt) * RS + (g * kHeadDim + 8 * c) * ESZ), v2);
            float p[G];
            load_p<G>(pw + tt * G, p);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
              const float2 pp = make_float2(p[hh], p[hh]);
#pragma unroll
              for (int e = 0; e < 4; ++e) o2[hh][e] = __ffma2_rn(v2[e], pp, o2[hh][e]);
            }
          }
        }
        __syncwarp();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot_i]);
    }

    // ---- finish the piece -----------------------------------------------------
    // Sum of p per head: the lanes of head hl in every token group.
#pragma unroll
    for (int off = 1; off < LPH; off <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, off);
#pragma unroll
    for (int off = D; off < 32; off <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, off);
    float lsum[G], mh[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      lsum[hh] = __shfl_sync(0xffffffffu, l_lane, head_lane(hh));
      mh[hh] = __shfl_sync(0xffffffffu, m_run, head_lane(hh));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o2[hh][e].x += __shfl_xor_sync(0xffffffffu, o2[hh][e].x, 16);
        o2[hh][e].y += __shfl_xor_sync(0xffffffffu, o2[hh][e].y, 16);
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      if ((G >= 2 ? (hh & 1) : 0) != half) continue;
      const int h = g * G + hh;
      if (whole) {
        const float inv = lsum[hh] > 0.f ? 1.f / lsum[hh] : 0.f;
        float f[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f[2 * e] = o2[hh][e].x * inv;
          f[2 * e + 1] = o2[hh][e].y * inv;
        }
        store8<IO>(obase + ((int64_t)r * a.hq + h) * kHeadDim + 8 * c, f);
      } else {
        const int64_t id = static_cast<int64_t>(blockIdx.x) + r;
        float* op = a.ws_o + (id * a.hq + h) * kHeadDim + 8 * c;
        *reinterpret_cast<float4*>(op) = make_float4(o2[hh][0].x, o2[hh][0].y, o2[hh][1].x, o2[hh][1].y);
        *reinterpret_cast<float4*>(op + 4) =
            make_float4(o2[hh][2].x, o2[hh][2].y, o2[hh][3].x, o2[hh][3].y);
        if (c == 0) a.ws_ml[id * a.hq + h] = make_float2(mh[hh], lsum[hh]);
      }
    }
  }
  }
}

// Merge the pieces of requests that spanned more than one CTA; zero the rows
// of empty contexts.  One warp per (request, q head); lane owns 4 dims.  The
// pieces' (max, sum) pairs are read in parallel across lanes and the partial
// rows with independent loads, so the merge costs a few memory round trips.
//
// Cascade mode (pre_ml != null): every request also has nsplit shared-prefix
// partials, [split][request][head], merged first; partials with sum 0 (empty
// ranges) are skipped, and the suffix pieces are merged even when there is
// only one.
template <typename E>
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ cum,
    const int64_t* __restrict__ per_p, const float2* __restrict__ ml, const float* __restrict__ o,
    int32_t hq, void* __restrict__ out, const float2* __restrict__ pre_ml,
    const float* __restrict__ pre_o, int32_t nsplit) {
  // Partials come from the split kernel launched just before this one.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int r = blockIdx.x;
  const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= hq) return;
  E* dst = static_cast<E*>(out) + ((int64_t)r * hq + h) * kHeadDim + 4 * lane;
  const int64_t c0 = cum[r], c1 = cum[r + 1];
  const bool cascade = pre_ml != nullptr;
  if (seq_lens[r] < 1 || (c1 <= c0 && !cascade)) {
    if constexpr (sizeof(E) == 2) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(0, 0);
    } else {
      *reinterpret_cast<float4*>(dst) = make_float4(0, 0, 0, 0);
    }
    return;
  }
  const int64_t per = *per_p;
  const int64_t k_lo = c1 > c0 ? c0 / per : 0, k_hi = c1 > c0 ? (c1 - 1) / per : -1;
  if (!cascade && k_lo == k_hi) return;  // written by its only piece
  // Online merge.  Partials are taken eight at a time, all of a batch's
  // loads ((max, sum) pairs and output slices, independent of each other)
  // issued before any merge, so a batch costs about one memory round trip.
  // Cascade mode merges the nsplit shared-prefix partials first.
  float M = -INFINITY, den = 0.f;
  float4 acc = make_float4(0, 0, 0, 0);
  auto merge = [&](float2 st, float4 x) {
    if (!(st.y > 0.f)) return;  // empty partial (its output slice is not read)
    const float Mn = fmaxf(M, st.x);
    const float wa = exp2f(M - Mn), wb = exp2f(st.x - Mn);
    den = den * wa + wb * st.y;
    acc.x = acc.x * wa + wb * x.x;
    acc.y = acc.y * wa + wb * x.y;
    acc.z = acc.z * wa + wb * x.z;
    acc.w = acc.w * wa + wb * x.w;
    M = Mn;
  };
  const int64_t B = gridDim.x;
  const int64_t npre = cascade ? nsplit : 0;
  const int64_t total = npre + (k_hi - k_lo + 1);
  constexpr int kBatch = 8;
  for (int64_t b0 = 0; b0 < total; b0 += kBatch) {
    float2 st[kBatch];
    float4 x[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t t = b0 + i;
      st[i] = make_float2(-INFINITY, 0.f);
      x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < total) {
        const bool pre = t < npre;
        const int64_t id = pre ? (t * B + r) * hq + h : (k_lo + (t - npre) + r) * hq + h;
        st[i] = (pre ? pre_ml : ml)[id];
        x[i] = *reinterpret_cast<const float4*>((pre ? pre_o : o) + id * kHeadDim + 4 * lane);
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) merge(st[i], x[i]);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  if constexpr (sizeof(E) == 2) {
    uint2 w;
    w.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    w.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(dst) = w;
  } else {
    *reinterpret_cast<float4*>(dst) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

// Tensor map of one pool plane for page-box stages (see tma_page_box): slot
// is the second dimension, so a box of 16 slots lands as 16 consecutive
// 128-byte rows per head (and half row), which the 128B swizzle spreads over
// all banks for the consumers' ldmatrix reads.
bool make_page_map(CUtensorMap* map, const uint8_t* base, int64_t num_slots, int64_t slot_stride, int hkv,
                   bool fp8) {
  auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_fn());
  if (fn == nullptr || num_slots < 16) return false;
  void* gaddr = const_cast<uint8_t*>(base);
  if (fp8) {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(num_slots), static_cast<cuuint64_t>(hkv)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(slot_stride), 128};
    cuuint32_t box[3] = {128, 16, static_cast<cuuint32_t>(hkv)};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, gaddr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(num_slots), 2, static_cast<cuuint64_t>(hkv)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(slot_stride), 128, 256};
  cuuint32_t box[4] = {64, 16, 2, static_cast<cuuint32_t>(hkv)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, gaddr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename E, int G, bool kPaged>
cudaError_t launch_split_t(const DecodeArgs& a, int grid, cudaStream_t s, const CascadeView* cv,
                           const CUtensorMap& kmap, const CUtensorMap& vmap) {
  constexpr int T = DecodeTraits<E>::kTokensPerStage;
  using LT = DecodeLayoutTraits<E>;
  constexpr int kPsm = LT::template psm_per_warp<G>();
  constexpr int kPad = kPaged ? 0 : LT::kRowPad;
  constexpr int kSlack = kPaged ? 1024 : 0;  // in-kernel 1024-byte alignment of the stages
  const DecodeSmem L = decode_smem_layout(a.batch, a.hkv, a.row_bytes + kPad, T, kPsm);
  // The limit is raised once to the largest layout any batch can need.
  static int smem_state[kMaxDevicesHost] = {};
  const int max_bytes =
      decode_smem_layout(kMaxBatch, 8, 8 * kHeadDim * static_cast<int>(sizeof(E)) + kPad, T, kPsm).total + kSlack;
  if (L.total + kSlack > max_bytes) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(decode_split_kernel<E, G, kPaged>, max_bytes, smem_state);
  if (e != cudaSuccess) return e;
  // Both kernels use programmatic dependent launch: the split kernel is
  // scheduled and sets up its barriers while the preceding kernel finishes,
  // and reads nothing (lengths, table, pool) before griddepcontrol.wait; the
  // combine kernel is scheduled while the split kernel runs and waits for
  // its partials.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * (LT::kProd + a.hkv));
  cfg.dynamicSmemBytes = L.total + kSlack;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_split_kernel<E, G, kPaged>, a, kmap, vmap);
  if (e != cudaSuccess) return e;
  if (cv != nullptr && cv->prefix_done != nullptr) {
    e = cudaStreamWaitEvent(s, cv->prefix_done, 0);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t ccfg = cfg;
  ccfg.gridDim = dim3(a.batch, (a.hq + 3) / 4);
  ccfg.blockDim = dim3(128);
  ccfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&ccfg, decode_combine_kernel<typename DecodeTraits<E>::IO>, a.seq_lens,
                            (const int32_t*)a.ws_cum,
                            (const int64_t*)a.ws_per, (const float2*)a.ws_ml, (const float*)a.ws_o,
                            a.hq, a.out, cv ? cv->pre_ml : nullptr, cv ? cv->pre_o : nullptr,
                            cv ? cv->nsplit : 0);
}

// Page sizes that are multiples of 16 take page-box stages (bf16 and FP8
// pools); every other pool streams token rows.
template <typename E, int G>
cudaError_t launch_decode_t(const DecodeArgs& a, int grid, cudaStream_t s, const CascadeView* cv) {
  if constexpr (DecodeLayoutTraits<E>::kMma) {
    if (a.page_size % 16 == 0) {
      CUtensorMap km, vm;
      if (make_page_map(&km, a.kbase, a.num_slots, a.slot_stride_bytes, a.hkv, sizeof(E) == 1) &&
          make_page_map(&vm, a.vbase, a.num_slots, a.slot_stride_bytes, a.hkv, sizeof(E) == 1))
        return launch_split_t<E, G, true>(a, grid, s, cv, km, vm);
    }
  }
  CUtensorMap none;
  memset(&none, 0, sizeof(none));
  return launch_split_t<E, G, false>(a, grid, s, cv, none, none);
}

}  // namespace

int decode_grid_size() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

size_t decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int grid) {
  const size_t pieces = static_cast<size_t>(grid) + static_cast<size_t>(batch);
  size_t b = 0;
  b += 16;                                               // per
  b += ((static_cast<size_t>(batch) + 1) * 4 + 15) & ~size_t(15);  // cum
  b += pieces * num_q_heads * sizeof(float2);            // (m, l)
  b = (b + 15) & ~size_t(15);
  b += pieces * num_q_heads * kHeadDim * sizeof(float);  // partial O
  return b;
}

cudaError_t launch_decode(const PoolView& pool, const TableView& t, const void* q,
                          int32_t num_q_heads, const int32_t* table_idx, const int32_t* seq_lens,
                          int32_t batch, float scale, void* out, void* workspace, int grid,
                          int32_t* err, cudaStream_t s, const CascadeView* cascade) {
  if (batch == 0) return cudaSuccess;
  DecodeArgs a;
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
  a.seq_lens = seq_lens;
  a.batch = batch;
  a.q = q;
  a.out = out;
  a.hq = num_q_heads;
  a.hkv = pool.num_kv_heads;
  a.scale_log2 = scale * kLog2e * pool.k_scale;
  a.v_scale = pool.v_scale;
  a.row_bytes = pool.num_kv_heads * kHeadDim * pool.esize;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.ws_per = reinterpret_cast<int64_t*>(w);
  w += 16;
  a.ws_cum = reinterpret_cast<int32_t*>(w);
  w += ((static_cast<size_t>(batch) + 1) * 4 + 15) & ~size_t(15);
  const size_t pieces = static_cast<size_t>(grid) + static_cast<size_t>(batch);
  a.ws_ml = reinterpret_cast<float2*>(w);
  w += pieces * num_q_heads * sizeof(float2);
  w = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(w) + 15) & ~uintptr_t(15));
  a.ws_o = reinterpret_cast<float*>(w);
  a.err = err;
  a.kv_start = cascade ? cascade->kv_start : nullptr;
  a.cascade = cascade ? 1 : 0;
  const int G = num_q_heads / pool.num_kv_heads;
  if (pool.dtype == PKV_DTYPE_FP8_E4M3) {
    switch (G) {
      case 1: return launch_decode_t<__nv_fp8_e4m3, 1>(a, grid, s, cascade);
      case 2: return launch_decode_t<__nv_fp8_e4m3, 2>(a, grid, s, cascade);
      case 4: return launch_decode_t<__nv_fp8_e4m3, 4>(a, grid, s, cascade);
      case 8: return launch_decode_t<__nv_fp8_e4m3, 8>(a, grid, s, cascade);
      case 16: return launch_decode_t<__nv_fp8_e4m3, 16>(a, grid, s, cascade);
    }
  } else if (pool.dtype == PKV_DTYPE_BF16) {
    switch (G) {
      case 1: return launch_decode_t<__nv_bfloat16, 1>(a, grid, s, cascade);
      case 2: return launch_decode_t<__nv_bfloat16, 2>(a, grid, s, cascade);
      case 4: return launch_decode_t<__nv_bfloat16, 4>(a, grid, s, cascade);
      case 8: return launch_decode_t<__nv_bfloat16, 8>(a, grid, s, cascade);
      case 16: return launch_decode_t<__nv_bfloat16, 16>(a, grid, s, cascade);
    }
  } else {
    switch (G) {
      case 1: return launch_decode_t<float, 1>(a, grid, s, cascade);
      case 2: return launch_decode_t<float, 2>(a, grid, s, cascade);
      case 4: return launch_decode_t<float, 4>(a, grid, s, cascade);
      case 8: return launch_decode_t<float, 8>(a, grid, s, cascade);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace pkv
