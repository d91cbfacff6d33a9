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
//  * Warp 0 is the producer: for each stage of 16 tokens it translates the
//    tokens' slots through the page table and issues one 1-D bulk copy
//    (cp.async.bulk, the TMA's non-tensor form) per token and plane.  A token
//    row holds all KV heads of the slot (2 KB for 8 heads x 128 x bf16), so
//    every copy is a long contiguous read.  Stages live in a 3-deep ring of
//    shared memory guarded by full/empty mbarriers.
//  * Warps 1..Hkv are consumers, one per KV head.  Lane = (half, c): c picks
//    8 consecutive dims, half picks even/odd tokens.  Scores for 8 tokens x G
//    heads are reduced across the 16 lanes of a half with a transposing
//    butterfly (each step halves the values a lane keeps), so the reduction
//    costs about one shuffle per (token, head) instead of four.  Softmax runs
//    in the log2 domain with exp2 and a lazily moved running max (the
//    accumulators are rescaled only when the max grows by more than 2^8).
//    PV accumulates with packed f32x2 FMAs.
//  * A piece that covers a whole request writes the final output; other
//    pieces write an un-normalised fp32 partial plus (max, sum) to the
//    workspace and decode_combine_kernel merges them.
//  * Cascade suffix pass (cascade.cu): each request starts at its own table
//    column, every piece writes a partial, and the combine kernel also merges
//    the shared-prefix partials.
//  * FP8 (E4M3) pools: 32 tokens per stage (1 KB rows); codes widen exactly to
//    half and then float; the K scale is folded into the softmax scale and
//    the V scale into the output.
#include <cuda_bf16.h>

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

// Shared memory layout (bytes), identical on host and device.
struct DecodeSmem {
  int32_t cum_off, psm_off, ring_off, stage_bytes, total;
};

__host__ __device__ inline DecodeSmem decode_smem_layout(int batch, int hkv, int row_bytes, int T,
                                                         int G) {
  DecodeSmem L;
  int off = 2 * kStages * 8 + 16;  // full/empty barriers + abort flag
  L.cum_off = off;
  off += 4 * (batch + 1);
  off = (off + 15) & ~15;
  L.psm_off = off;
  off += 4 * hkv * T * G;
  off = (off + 127) & ~127;
  L.ring_off = off;
  L.stage_bytes = 2 * T * row_bytes;
  L.total = off + kStages * L.stage_bytes;
  return L;
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

// 16 consecutive E4M3 codes (one 16-byte shared-memory load) -> two groups of
// 8 floats (exact: code -> half -> float).
__device__ __forceinline__ void load16_e4m3(const uint8_t* p, float2 (&lo)[4], float2 (&hi)[4]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] & 0xffffu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u[i] >> 16), __NV_E4M3);
    float2 (&dst)[4] = i < 2 ? lo : hi;
    dst[(2 * i) & 3] = __half22float2(*reinterpret_cast<const __half2*>(&a));
    dst[(2 * i + 1) & 3] = __half22float2(*reinterpret_cast<const __half2*>(&b));
  }
}

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

template <typename E, int G>
__global__ void __launch_bounds__(32 * 9, 1) decode_split_kernel(const DecodeArgs a) {
  constexpr int T = DecodeTraits<E>::kTokensPerStage;
  constexpr int SUB = (64 / G < T) ? 64 / G : T;  // tokens per softmax sub-step
  constexpr int HALF = SUB / 2;                    // PV: tokens per lane per sub-step
  // Scores: D lanes share a token (each owns 16/D units of 8 dims), TL =
  // 32/D tokens are in flight per warp step, and a lane keeps V = SPL*G
  // partial sums per sub-step.  D = 8 halves the reduction of D = 16; wide
  // groups (G = 8, whose q would not fit in registers) keep D = 16.  A lane's
  // units are dims 8d and 64 + 8d (16-byte loads of bf16 or fp32 rows), or,
  // for FP8 rows, the 16 consecutive dims 16d .. 16d + 15, read as one
  // 16-byte load (so that the 8 lanes of a token read 128 contiguous bytes).
  constexpr int D = G >= 8 ? 16 : 8;
  constexpr bool kWideFp8 = sizeof(E) == 1 && D == 8;
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

  extern __shared__ __align__(128) uint8_t smem[];
  // Let the combine kernel be scheduled early; it waits for this grid anyway.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncons = a.hkv;
  const DecodeSmem L = decode_smem_layout(a.batch, a.hkv, a.row_bytes, T, G);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(empty + kStages);
  int32_t* cum = reinterpret_cast<int32_t*>(smem + L.cum_off);
  float* psm = reinterpret_cast<float*>(smem + L.psm_off);
  uint8_t* ring = smem + L.ring_off;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
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

  if (warp == 0) {
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
      uint8_t* vst = kst + T * a.row_bytes;
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
      const bool load = in_piece && slot >= 0;
      if (in_piece && !load) {
        // Out-of-range entry: the row reads as zeros (error already flagged).
        for (int b = 0; b < a.row_bytes; b += 16) {
          *reinterpret_cast<uint4*>(kst + lane * a.row_bytes + b) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(vst + lane * a.row_bytes + b) = make_uint4(0, 0, 0, 0);
        }
        // Later bulk copies (async proxy) may write these bytes again.
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      const unsigned nload = __popc(__ballot_sync(0xffffffffu, load));
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[slot_i], nload * 2u * a.row_bytes);
      __syncwarp();
      if (load) {
        bulk_g2s(kst + lane * a.row_bytes, a.kbase + slot * a.slot_stride_bytes, a.row_bytes,
                 &full[slot_i], policy);
        bulk_g2s(vst + lane * a.row_bytes, a.vbase + slot * a.slot_stride_bytes, a.row_bytes,
                 &full[slot_i], policy);
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
    return;
  }

  // ============================= consumers ==================================
  // Scores use the token-group lane map (tl, d) = (lane / D, lane % D); the
  // PV product uses (half, c) = (lane / 16, lane % 16): lane c owns dims
  // 8c .. 8c+7 and half picks even or odd tokens.  The p values pass from the
  // first map to the second through the warp's p buffer [SUB][G].
  const int g = warp - 1;  // KV head
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
  auto unit_dim = [&](int m) { return kWideFp8 ? 16 * d + 8 * m : 8 * (d + D * m); };
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
      const uint8_t* vst = kst + T * a.row_bytes;

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
          if constexpr (kWideFp8) {
            load16_e4m3(kst + t * a.row_bytes + g * kHeadDim + 16 * d, kw[0], kw[UPL - 1]);
          } else {
#pragma unroll
            for (int m = 0; m < UPL; ++m)
              load8<E>(reinterpret_cast<const E*>(kst + t * a.row_bytes + (g * kHeadDim + unit_dim(m)) * ESZ),
                       kw[m]);
          }
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
            load8<E>(reinterpret_cast<const E*>(vst + (sub + tt) * a.row_bytes + (g * kHeadDim + 8 * c) * ESZ), v2);
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
    if constexpr (sizeof(E) == 1) {  // FP8 pool: V codes stand for code * v_scale
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o2[hh][e].x *= a.v_scale;
          o2[hh][e].y *= a.v_scale;
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
  // Online merge: the loads of consecutive pieces are independent, so the
  // unrolled loops keep several in flight.
  float M = -INFINITY, den = 0.f;
  float4 acc = make_float4(0, 0, 0, 0);
  auto merge = [&](float2 st, const float* src) {
    if (!(st.y > 0.f)) return;  // empty partial
    const float4 x = *reinterpret_cast<const float4*>(src + 4 * lane);
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
#pragma unroll 4
  for (int sp = 0; sp < nsplit; ++sp) {
    const int64_t id = (sp * B + r) * hq + h;
    merge(pre_ml[id], pre_o + id * kHeadDim);
  }
#pragma unroll 4
  for (int64_t k = k_lo; k <= k_hi; ++k) merge(ml[(k + r) * hq + h], o + ((k + r) * hq + h) * kHeadDim);
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

template <typename E, int G>
cudaError_t launch_decode_t(const DecodeArgs& a, int grid, cudaStream_t s, const CascadeView* cv) {
  constexpr int T = DecodeTraits<E>::kTokensPerStage;
  const DecodeSmem L = decode_smem_layout(a.batch, a.hkv, a.row_bytes, T, G);
  // The limit is raised once to the largest layout any batch can need.
  static int smem_state[kMaxDevicesHost] = {};
  const int max_bytes = decode_smem_layout(kMaxBatch, 8, 8 * kHeadDim * static_cast<int>(sizeof(E)), T, G).total;
  if (L.total > max_bytes) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(decode_split_kernel<E, G>, max_bytes, smem_state);
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
  cfg.blockDim = dim3(32 * (1 + a.hkv));
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_split_kernel<E, G>, a);
  if (e != cudaSuccess) return e;
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
    }
  } else if (pool.dtype == PKV_DTYPE_BF16) {
    switch (G) {
      case 1: return launch_decode_t<__nv_bfloat16, 1>(a, grid, s, cascade);
      case 2: return launch_decode_t<__nv_bfloat16, 2>(a, grid, s, cascade);
      case 4: return launch_decode_t<__nv_bfloat16, 4>(a, grid, s, cascade);
      case 8: return launch_decode_t<__nv_bfloat16, 8>(a, grid, s, cascade);
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
