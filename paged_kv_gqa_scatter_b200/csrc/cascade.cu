// Cascade (shared-prefix aware) decode.
//
// What it computes: the same decode attention as decode.cu -- each request's
// one query token over its whole context -- for batches in which groups of
// requests share a radix-cached prefix ("Mini-SGLang 完整剖析",
// blog.rzhang-lab.cn/post/3, §1.4: requests with a common prefix reuse the
// same KV pages).  Softmax attention over a union of disjoint key sets is the
// (max, sum)-weighted merge of the attention over each set, so the context is
// cut at the shared-prefix boundary:
//
//  1. cascade_prep_kernel: request r of group g gets kv_start[r] = p_g, the
//     group's shared prefix length (validated against its context length).
//  2. The shared prefix, once per group: every member's query rows together
//     form the M dimension of the tcgen05 extend kernel in prefix mode
//     (extend_tc.cu), which reads the prefix's K/V tiles once per group and
//     KV head instead of once per request, and writes fp32 partials.  The
//     prefix keys are cut into nsplit ranges so the pass fills the GPU.
//  3. The per-request suffix (columns p_g .. seq_len - 1) by the split-KV
//     decode kernel, every piece writing a partial.
//  4. decode_combine_kernel merges the prefix partials and suffix pieces.
//
// Work moved: the prefix costs 4 d Hq p_g FLOPs per member on the tensor
// cores and p_g x 4 KB of HBM reads per group (Hkv 8, bf16), instead of
// p_g x 4 KB per member through the memory pipe.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

// One thread per request: find its group (largest g with offsets[g] <= r),
// check the group structure and the prefix length, write kv_start.
__global__ void __launch_bounds__(256) cascade_prep_kernel(const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ prefix,
                                                           int32_t groups,
                                                           const int32_t* __restrict__ seq_lens,
                                                           int32_t batch, int64_t capacity,
                                                           int32_t* __restrict__ kv_start,
                                                           int32_t* err) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < groups && off[r] > off[r + 1]) set_err(err, PKV_DEV_ERR_BAD_LENGTH);
  if (r == 0 && (off[0] != 0 || off[groups] != batch)) set_err(err, PKV_DEV_ERR_BAD_LENGTH);
  if (r >= batch) return;
  int l = 0, h = groups;  // invariant: off[l] <= r < off[h] when the offsets are valid
  while (h - l > 1) {
    const int m = (l + h) >> 1;
    if (off[m] <= r) l = m; else h = m;
  }
  int64_t p = prefix[l];
  const int32_t n = seq_lens[r];
  if (p < 0 || p > n || p > capacity) {
    set_err(err, PKV_DEV_ERR_BAD_LENGTH);
    p = p < 0 ? 0 : p;
    p = p > n ? (n < 0 ? 0 : n) : p;
    p = p > capacity ? capacity : p;
  }
  kv_start[r] = static_cast<int32_t>(p);
}

struct CascadeLayout {
  int32_t nsplit, split_keys;
  size_t start_off, ml_off, o_off, decode_off, total;
};

}  // namespace

// Prefix ranges of about 1024 keys (at most 16): enough CTAs to fill the GPU
// when one group shares a 4k prefix, few enough partials to merge cheaply.
static CascadeLayout cascade_layout(int32_t batch, int32_t hq, int64_t max_prefix, int grid) {
  CascadeLayout L;
  constexpr int64_t kKeysPerSplit = 1024, kMaxSplits = 16, kStep = 64;
  const int64_t ns = max_prefix <= 0 ? 0 : std::min(kMaxSplits, (max_prefix + kKeysPerSplit - 1) / kKeysPerSplit);
  L.nsplit = static_cast<int32_t>(ns);
  const int64_t per = ns == 0 ? 0 : (max_prefix + ns - 1) / ns;
  L.split_keys = static_cast<int32_t>((per + kStep - 1) / kStep * kStep);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = static_cast<size_t>(ns) * batch * hq;
  L.start_off = 0;
  L.ml_off = up(static_cast<size_t>(batch) * 4);
  L.o_off = L.ml_off + up(rows * sizeof(float2));
  L.decode_off = L.o_off + up(rows * kHeadDim * sizeof(float));
  L.total = L.decode_off + decode_workspace_bytes(batch, hq, grid);
  return L;
}

size_t cascade_workspace_bytes(int32_t batch, int32_t num_q_heads, int64_t max_prefix_len) {
  return cascade_layout(batch, num_q_heads, max_prefix_len, decode_grid_size()).total;
}

cudaError_t launch_cascade_prep(const int32_t* group_offsets, const int32_t* group_prefix,
                                int32_t num_groups, const int32_t* seq_lens, int32_t batch,
                                int64_t prefix_capacity, int32_t* kv_start, int32_t* err,
                                cudaStream_t s) {
  const int n = std::max(batch, num_groups);
  cascade_prep_kernel<<<(n + 255) / 256, 256, 0, s>>>(group_offsets, group_prefix, num_groups, seq_lens,
                                                      batch, prefix_capacity, kv_start, err);
  return cudaGetLastError();
}

// The prefix pass (tensor cores) and the suffix pass (HBM) use different
// units, so when the prefix pass is small enough they run side by side: the
// prefix pass on an auxiliary stream with about 43% of the SMs' worth of
// CTAs, the suffix pass on the caller's stream with the remaining SMs as its
// persistent grid, joined by an event before the merge.  (Inside a CUDA graph
// the fork and join become graph edges.)  The auxiliary stream and events
// are created once per device on the first call made outside stream capture;
// until then, and whenever the prefix grid would take more than half the
// SMs, the two passes run one after the other on the caller's stream.
namespace {

struct AuxStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  // Held from the fork record to the join wait, so that calls from several
  // host threads cannot interleave their records of the shared events.
  std::mutex mu;
};
AuxStream g_aux[kMaxDevicesHost];

AuxStream* aux_stream(cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesHost) return nullptr;
  AuxStream& a = g_aux[dev];
  std::lock_guard<std::mutex> lock(a.mu);  // released before the caller locks it again
  if (a.join != nullptr) return &a;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
  if (a.stream == nullptr && cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking) != cudaSuccess) {
    a.stream = nullptr;
    return nullptr;
  }
  if (a.fork == nullptr && cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess) {
    a.fork = nullptr;
    return nullptr;
  }
  if (cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess) {
    a.join = nullptr;
    return nullptr;
  }
  return &a;
}

constexpr double kPrefixShare = 0.43;  // share of the SMs the side-by-side prefix pass gets

}  // namespace

cudaError_t launch_decode_cascade(const PoolView& pool, const TableView& t, const void* q,
                                  int32_t num_q_heads, const int32_t* table_idx,
                                  const int32_t* seq_lens, int32_t batch,
                                  const int32_t* group_offsets, const int32_t* group_prefix,
                                  int32_t num_groups, int64_t max_prefix_len, float scale, void* out,
                                  void* workspace, int32_t* err, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  const int sms = decode_grid_size();
  const CascadeLayout L = cascade_layout(batch, num_q_heads, max_prefix_len, sms);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int32_t* kv_start = reinterpret_cast<int32_t*>(w + L.start_off);
  float2* pre_ml = reinterpret_cast<float2*>(w + L.ml_off);
  float* pre_o = reinterpret_cast<float*>(w + L.o_off);
  // Prefix-pass CTAs per key split: KV heads x query blocks (two 128-row Q
  // tiles of 128 / G tokens) x groups.
  const int G = num_q_heads / pool.num_kv_heads;
  const int64_t per_split = static_cast<int64_t>(pool.num_kv_heads) * ((batch + 2 * (128 / G) - 1) / (2 * (128 / G))) *
                            num_groups;
  int32_t nsplit = L.nsplit, split_keys = L.split_keys;
  AuxStream* aux = nullptr;
  if (L.nsplit > 0 && per_split > 0 && per_split <= kPrefixShare * sms) {
    int64_t ns = std::llround(kPrefixShare * sms / static_cast<double>(per_split));
    ns = std::max<int64_t>(1, std::min<int64_t>(ns, L.nsplit));
    if (per_split * ns <= sms / 2) {
      aux = aux_stream(s);
      if (aux != nullptr) {
        nsplit = static_cast<int32_t>(ns);
        const int64_t per = (max_prefix_len + nsplit - 1) / nsplit;
        split_keys = static_cast<int32_t>((per + 63) / 64 * 64);
      }
    }
  }
  const int64_t capacity = static_cast<int64_t>(nsplit) * split_keys;
  cudaError_t e = launch_cascade_prep(group_offsets, group_prefix, num_groups, seq_lens, batch, capacity,
                                      kv_start, err, s);
  if (e != cudaSuccess) return e;
  if (aux == nullptr) {
    e = launch_extend_prefix(pool, t, q, num_q_heads, table_idx, group_offsets, group_prefix, num_groups, batch,
                             nsplit, split_keys, scale, pre_ml, pre_o, err, s);
    if (e != cudaSuccess) return e;
    CascadeView cv{kv_start, pre_ml, pre_o, nsplit, nullptr};
    return launch_decode(pool, t, q, num_q_heads, table_idx, seq_lens, batch, scale, out, w + L.decode_off, sms,
                         err, s, &cv);
  }
  // Side by side: fork the auxiliary stream after the prep kernel, run the
  // prefix pass there and the suffix pass here on the SMs it leaves free.
  std::lock_guard<std::mutex> lock(aux->mu);
  e = cudaEventRecord(aux->fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(aux->stream, aux->fork, 0);
  if (e != cudaSuccess) return e;
  e = launch_extend_prefix(pool, t, q, num_q_heads, table_idx, group_offsets, group_prefix, num_groups, batch,
                           nsplit, split_keys, scale, pre_ml, pre_o, err, aux->stream);
  if (e == cudaSuccess) e = cudaEventRecord(aux->join, aux->stream);
  if (e != cudaSuccess) return e;
  const int suffix_grid = static_cast<int>(sms - per_split * nsplit);
  CascadeView cv{kv_start, pre_ml, pre_o, nsplit, aux->join};
  return launch_decode(pool, t, q, num_q_heads, table_idx, seq_lens, batch, scale, out, w + L.decode_off,
                       suffix_grid, err, s, &cv);
}

}  // namespace pkv
