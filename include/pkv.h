/*
 * pkv.h -- C ABI of the paged KV pool attention library (sm_100a / B200).
 *
 * The library implements the GPU hot path of a mini-SGLang-style serving
 * engine: scattering each step's new K/V rows into a paged pool, and GQA
 * attention over that pool through a token-granular page table, for decode
 * (one query token per request) and for extend (a prefill chunk attending
 * causally to its cached prefix and to itself).
 *
 * Sources (web pages on mini-SGLang, cited by title and section):
 *   [P5] "Mini-SGLang 完整剖析" (blog.rzhang-lab.cn/post/3)
 *        §1.2 prefill vs decode, §1.3 KV cache, §1.4 paged pool and prefix
 *        sharing, §4.2.3 request length fields, §4.4.3 pool tensor,
 *        §4.5.6 shared RotaryEmbedding, §4.6.4 page-table metadata,
 *        §4.6.6 CUDA-graph capture, §4.6.7 attention layer / store_kv,
 *        §4.9.4 store kernel shape checks.
 *   [P4] "深入解析 mini-sglang" (yunpan.plus), chunked prefill.
 *   [P3] "mini-sglang 深度分析报告" (nightvoyager.top), design notes
 *        (page_size-1 page table).
 *
 * Conventions shared by every call
 * --------------------------------
 * Ownership: the caller owns every buffer passed in (device memory unless a
 *   parameter says "host").  No call keeps a pointer after it returns, and no
 *   compute call allocates device memory; scratch space comes from a
 *   caller-provided workspace whose size a *_workspace_bytes query returns,
 *   or from a pkv_workspace object (the only calls that allocate).
 * Streams: every compute call is asynchronous on the given stream (0 = the
 *   legacy default stream) and never synchronises the host.
 * Errors: calls return a pkv_status.  Host-side checks (null pointers,
 *   negative sizes, unsupported dtype or head_dim, misaligned strides, a
 *   workspace that is too small) return an error before anything is
 *   launched.  Data-dependent faults found on the device (a slot or page
 *   table index out of range, an empty context) are not trapped: the
 *   offending element is skipped or zero-filled, and a bit from
 *   pkv_device_error is OR-ed into the caller's `dev_err` word (a device
 *   int32, may be NULL).  No kernel traps, asserts or waits without bound:
 *   each internal wait gives up after about one second and sets
 *   PKV_DEV_ERR_TIMEOUT.
 * Element types: bf16 (the product path), fp32 (a check build of the same
 *   kernels for tighter numerical comparison; no cascade decode) and a
 *   scaled FP8 E4M3 pool (every call; see pkv_pool).  head_dim must be 128.
 * Launch overlap: the store calls let the next kernel launch early
 *   (programmatic dependent launch); decode waits for the preceding kernel
 *   before it reads any input, so inputs written by that kernel are safe.
 * CUDA graphs: every compute call can be captured; make the first call on
 *   a device outside capture (it sets kernel attributes once).
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* pkv_stream_t; /* a cudaStream_t */

typedef enum {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad stride   */
  PKV_ERR_UNSUPPORTED = 2,      /* dtype, head_dim or head counts not built  */
  PKV_ERR_MISALIGNED = 3,       /* a pointer or stride breaks 16-byte rules  */
  PKV_ERR_WORKSPACE = 4,        /* workspace missing or too small            */
  PKV_ERR_CUDA = 5,             /* a CUDA runtime call failed                */
  PKV_ERR_TOO_LARGE = 6         /* a size beyond a documented maximum        */
} pkv_status;

typedef enum {
  PKV_DEV_ERR_SLOT_RANGE = 1,    /* a slot (out_loc or table entry) >= num_slots or < 0 */
  PKV_DEV_ERR_TABLE_RANGE = 2,   /* table_idx row or column beyond the table            */
  PKV_DEV_ERR_EMPTY_CONTEXT = 4, /* decode seq_len < 1, or queries with no key          */
  PKV_DEV_ERR_BAD_LENGTH = 8,    /* negative prefix/extend length, or q_offsets broken  */
  PKV_DEV_ERR_PAGE_ALIGN = 16,   /* page_size > 1 and a page's first entry % page_size  */
  PKV_DEV_ERR_TIMEOUT = 32,      /* an internal wait gave up (never expected)           */
  PKV_DEV_ERR_POSITION = 64      /* a RoPE position outside [0, max_position)           */
} pkv_device_error;

typedef enum { PKV_DTYPE_BF16 = 0, PKV_DTYPE_F32 = 1, PKV_DTYPE_FP8_E4M3 = 2 } pkv_dtype;

/*
 * The KV pool [P5 §4.4.3; §1.4].
 *
 * The pages store K and V in one tensor (2, layers, pages, page_size,
 * kv_heads, head_dim) and address it flattened to slots (pages*page_size,
 * kv_heads, head_dim).  Here K and V are two planes with the same geometry,
 * each [num_layers][num_slots][num_kv_heads][head_dim], head_dim contiguous
 * and kv heads adjacent within a slot; `layer_stride` and `slot_stride` are
 * element strides between consecutive layers and slots (slot_stride >=
 * num_kv_heads*head_dim).  Slot s of page p and offset o is s = p*page_size
 * + o.  `k` and `v` must be 16-byte aligned and slot_stride*element_size a
 * multiple of 16.  The caller owns the planes.
 *
 * FP8 pool (dtype PKV_DTYPE_FP8_E4M3; not on the pages, which keep K/V in
 * the model dtype): each plane element is an OCP E4M3 code (1 byte) standing
 * for code_value * k_scale (K plane) or * v_scale (V plane).  Calls that
 * write the pool take bf16 rows and store the code of x * (1 / scale)
 * (float32 product, round to nearest even, saturated to +-448); decode,
 * cascade decode and extend read the codes (extend widens them to f16 for
 * the tensor cores) and take q and return out in bf16.  The scales must be
 * finite and > 0; they are ignored for the other dtypes.
 */
typedef struct {
  void* k;
  void* v;
  int64_t num_layers;
  int64_t num_slots;
  int64_t layer_stride;
  int64_t slot_stride;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t dtype; /* pkv_dtype */
  float k_scale;  /* FP8 pools: dequantisation scale of the K plane */
  float v_scale;  /* FP8 pools: dequantisation scale of the V plane */
} pkv_pool;

/*
 * The page table [P5 §4.6.4; P3 design notes].
 *
 * int32 [rows][cols] with row stride `row_stride` (elements), token
 * granular: entry [row][j] is the slot of token j of the request that owns
 * row `row`.  With page_size P > 1 the kernels follow the slice-and-divide
 * reading of the pages: the page of token j is entry [row][P*(j/P)] / P and
 * its slot is page*P + j%P (so only each page's first entry is read; it must
 * be a multiple of P).  `table_idx[r]` (int32, one per request) selects the
 * row of request r [P5 §6.1 table_idx; P4 chunked prefill: all chunks of a
 * request share one row].
 */
typedef struct {
  const int32_t* entries;
  int64_t rows;
  int64_t cols;
  int64_t row_stride;
} pkv_page_table;

/* Returns a static, human-readable string for a pkv_status or device-error bit set. */
const char* pkv_status_string(int status);

/* Library version string (static). */
const char* pkv_version(void);

/*
 * store_kv [P5 §4.6.7: the backend first scatters the step's new K/V into
 * the pool at batch.out_loc; §4.9.4: k/v are [L, D] with a row stride,
 * indices are int32 or int64, the pool rows are [-1, D]].
 *
 *   pool.k[layer][out_loc[i]][:] = k[i*k_row_stride .. + Hkv*head_dim)
 *   pool.v[layer][out_loc[i]][:] = v[i*v_row_stride .. + Hkv*head_dim)
 *   for 0 <= i < n_tokens, as a bit copy in the pool's element type (for an
 *   FP8 pool: the E4M3 codes of the bf16 rows, see pkv_pool).
 *
 * k, v: device, element type = pool.dtype (bf16 for an FP8 pool), row
 *   strides in elements (k and v are typically column slices of a fused qkv
 *   output); both pointers and strides must keep rows 16-byte aligned.
 * out_loc: device, int32 (out_loc_is_i64 = 0) or int64 (= 1), n_tokens entries.
 *   Slots must be distinct within one call (the pages give every new token
 *   its own slot); an out-of-range slot is skipped and sets
 *   PKV_DEV_ERR_SLOT_RANGE.
 * n_tokens == 0 is a no-op.
 */
int pkv_store_kv(const pkv_pool* pool, int32_t layer, const void* k, int64_t k_row_stride,
                 const void* v, int64_t v_row_stride, const void* out_loc,
                 int32_t out_loc_is_i64, int64_t n_tokens, int32_t* dev_err,
                 pkv_stream_t stream);

/*
 * qk_norm_rope_store -- q/k RMSNorm, RoPE and store_kv in one pass over the
 * rows of the fused qkv projection [P5 §4.6.7: the attention layer splits
 * qkv, applies q_norm / k_norm per head (Qwen3), rotates q and k in place at
 * the batch positions, then the backend stores k and v at out_loc; §4.5.6:
 * one shared RotaryEmbedding holds a cos_sin_cache of max_position x
 * rotary_dim].
 *
 *   for token t < n_tokens, with x = qkv row t = [q heads | k heads | v heads]:
 *     q_out[t][h]                  = rope(norm(q_h, q_norm_weight), pos[t])
 *     pool.k[layer][out_loc[t]][g] = rope(norm(k_g, k_norm_weight), pos[t])
 *     pool.v[layer][out_loc[t]][g] = v_g                      (bit copy)
 *   norm(x, w) = x / sqrt(mean(x^2) + eps) * w over the 128 dims (skipped
 *   when the weight pointer is NULL); rope is the rotate-half form over the
 *   whole head: for i < 64, (x_i, x_{i+64}) -> (x_i c - x_{i+64} s,
 *   x_{i+64} c + x_i s) with c, s = cos_sin_cache[pos][i], [pos][64 + i].
 *   The pages do not spell the pairing out; rotate-half is the reading taken.
 *
 * qkv: device, pool dtype (bf16 for an FP8 pool), rows of (Hq + 2 Hkv) * 128
 *   elements, row stride in elements; 16-byte aligned rows.
 * positions: device int32 (positions_is_i64 = 0) or int64 (= 1) [n_tokens];
 *   a position outside [0, max_position) zeroes that token's q and k rows and
 *   sets PKV_DEV_ERR_POSITION.
 * cos_sin_cache: device float32 [max_position][128] (64 cos then 64 sin),
 *   16-byte aligned.
 * q_norm_weight, k_norm_weight: device [128] in the qkv dtype, or NULL.
 * out_loc: as for pkv_store_kv (distinct slots; out of range is skipped and
 *   flagged).  q_out: device [n_tokens][num_q_heads][128], qkv dtype.
 * All arithmetic is fp32; outputs round to their type (nearest even; an FP8
 * pool stores the E4M3 codes of k * (1 / k_scale) and v * (1 / v_scale)).
 */
int pkv_qk_norm_rope_store(const pkv_pool* pool, int32_t layer, const void* qkv,
                           int64_t qkv_row_stride, int32_t num_q_heads, const void* positions,
                           int32_t positions_is_i64, const float* cos_sin_cache,
                           int64_t max_position, const void* q_norm_weight,
                           const void* k_norm_weight, float eps, const void* out_loc,
                           int32_t out_loc_is_i64, int64_t n_tokens, void* q_out,
                           int32_t* dev_err, pkv_stream_t stream);

/*
 * Workspace objects -- the one part of the library that allocates.  A caller
 * that does not want to size and own scratch memory creates one per stream
 * at start-up (before any CUDA-graph capture) on the current device:
 *
 *   pkv_workspace_create(max_batch, max_q_heads, max_prefix_len, &ws)
 *     allocates (cudaMalloc) a buffer large enough for pkv_decode_attn and
 *     pkv_decode_attn_cascade at up to max_batch requests of max_q_heads
 *     heads (cascade prefixes up to max_prefix_len; 0 if unused; extend
 *     needs no workspace) and a zeroed int32 device error word.
 *     PKV_ERR_CUDA if an allocation fails; *ws is NULL then.
 *   pkv_workspace_buffer(ws, &bytes) -> the buffer and its size, to pass as
 *     `workspace` / `workspace_bytes`.
 *   pkv_workspace_error_word(ws) -> the device error word, to pass as
 *     `dev_err`.
 *   pkv_read_device_error(ws, stream, &code) -> waits for the stream, stores
 *     the accumulated pkv_device_error bits in *code and clears the word.
 *   pkv_workspace_destroy(ws) frees both allocations (NULL is a no-op); no
 *     call that uses them may still be pending.
 *
 * The pages have no counterpart; their backends allocate such buffers once
 * when the engine starts.  A workspace must not be shared by calls that may
 * overlap on the GPU.
 */
typedef struct pkv_workspace pkv_workspace;
int pkv_workspace_create(int32_t max_batch, int32_t max_q_heads, int64_t max_prefix_len,
                         pkv_workspace** ws);
void pkv_workspace_destroy(pkv_workspace* ws);
void* pkv_workspace_buffer(const pkv_workspace* ws, size_t* bytes);
int32_t* pkv_workspace_error_word(const pkv_workspace* ws);
int pkv_read_device_error(pkv_workspace* ws, pkv_stream_t stream, int32_t* code);

/*
 * selftest_wait_timeout -- exercises the bounded wait of the pipelined
 * kernels.  The pages have no counterpart; it exists so that a test can
 * check, without faulting anything, that a wait nobody satisfies gives up.
 *
 * Launches one 32-thread kernel that waits on a shared-memory mbarrier that
 * nothing signals, with the same wait routine decode and extend use.  After
 * about one second the wait gives up, PKV_DEV_ERR_TIMEOUT is OR-ed into
 * *dev_err (device int32, required), and the kernel returns; the stream and
 * context remain usable.  Asynchronous like every other call.
 */
int pkv_selftest_wait_timeout(int32_t* dev_err, pkv_stream_t stream);

/*
 * gather_kv -- copies requests' K/V rows, in token order, through the page
 * table into dense buffers [P5 §4.6.4 page-table translation].  It is the
 * translation step the attention kernels perform internally, exposed on its
 * own so that it can be checked bit for bit.
 *
 *   k_out[row_offsets[r] + j][:] = pool.k[layer][slot(r, j)][:]  (same for v)
 *   for 0 <= j < seq_lens[r], 0 <= r < batch.
 *
 * table_idx, seq_lens: device int32 [batch]; row_offsets: device int64
 * [batch+1] (exclusive prefix sum of seq_lens, computed by the caller);
 * k_out, v_out: device, [row_offsets[batch]][Hkv*head_dim], pool dtype.
 * A slot out of range zero-fills the row and sets PKV_DEV_ERR_SLOT_RANGE.
 */
int pkv_gather_kv(const pkv_pool* pool, int32_t layer, const pkv_page_table* table,
                  const int32_t* table_idx, const int32_t* seq_lens, const int64_t* row_offsets,
                  int32_t batch, void* k_out, void* v_out, int32_t* dev_err,
                  pkv_stream_t stream);

/*
 * decode_attn [P5 §1.2: decode processes one token per request and is
 * memory-bandwidth bound; §4.6.4: cache_seqlens is each request's total KV
 * length; §4.6.7: store_kv runs before the kernel, so the context includes
 * the token just stored; §4.5.3: KV heads are shared by Hq/Hkv query heads].
 *
 *   out[r][h][:] = sum_j softmax_j(scale * q[r][h] . K_r[j][h/G]) V_r[j][h/G]
 *   over j < seq_lens[r], G = num_q_heads / pool.num_kv_heads,
 *   K_r[j] = pool.k[layer][slot(r, j)], V_r likewise.
 *
 * q: device [batch][num_q_heads][head_dim] contiguous, pool dtype (bf16 for
 *   an FP8 pool, whose K/V are read as code * scale).
 * out: device [batch][num_q_heads][head_dim] contiguous, q's dtype
 *   (fp32 accumulation, rounded to nearest-even on store).  bf16 and FP8
 *   pools compute on tensor cores: the softmax weights enter the PV product
 *   as two bf16 terms (bf16 pools, about 16 significant bits) or rounded to
 *   f16 (FP8 pools); fp32 pools stay fp32.
 * table_idx, seq_lens: device int32 [batch].
 * scale: softmax scale (the pages do not state it; 1/sqrt(head_dim) is the
 *   usual choice).
 * workspace: device scratch of at least pkv_decode_workspace_bytes(batch,
 *   num_q_heads) bytes, 16-byte aligned, owned by the caller, not shared by
 *   calls that may overlap on the GPU.
 * Supported: head_dim 128, num_kv_heads 1..8, num_q_heads/num_kv_heads in
 *   {1, 2, 4, 8}, and 16 on bf16 and FP8 pools (extend and cascade decode
 *   stop at 8).  seq_lens[r] < 1 writes a zero row and sets
 *   PKV_DEV_ERR_EMPTY_CONTEXT.  batch == 0 is a no-op.
 * The work is split across the context (split-KV): one persistent grid
 * walks (request, chunk) items, then a second kernel merges the chunks of
 * requests that had more than one.
 */
size_t pkv_decode_workspace_bytes(int32_t batch, int32_t num_q_heads);
int pkv_decode_attn(const pkv_pool* pool, int32_t layer, const void* q, int32_t num_q_heads,
                    const pkv_page_table* table, const int32_t* table_idx,
                    const int32_t* seq_lens, int32_t batch, float scale, void* out,
                    void* workspace, size_t workspace_bytes, int32_t* dev_err,
                    pkv_stream_t stream);

/*
 * decode_attn_noalloc -- the same decode as pkv_decode_attn for callers that
 * cannot allocate device memory.  The pages have no counterpart to this call.
 *
 * Who needs it: an engine that gives almost all free device memory to its KV
 * pool when it starts has no room left to allocate a workspace, and code
 * hosted by a framework that owns every device allocation may have no way to
 * allocate at all.  This call takes the same arguments as pkv_decode_attn
 * minus the workspace; its scratch is a fixed 16 MiB array inside the library
 * (pkv_decode_noalloc_max_scratch_bytes()), present on every device that
 * loads the library until the process exits.
 *
 * Limits and behaviour:
 *  - Returns PKV_ERR_TOO_LARGE, launching nothing, when
 *    pkv_decode_workspace_bytes(batch, num_q_heads) exceeds that size.
 *  - Every call made outside stream capture (with its device current) looks
 *    up the array's device address and caches it per device; a call made
 *    while its stream is captured reuses the cached address.  Make the first
 *    call on a device outside any stream capture, and, after a device reset
 *    (which reloads the library's device code and may move the array), make
 *    one more uncaptured call before capturing again.
 *  - All calls on a device share the array: calls that can overlap on the GPU
 *    (unordered streams) race; calls ordered on one stream are safe.  Nothing
 *    in the array needs to start at zero.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
size_t pkv_decode_noalloc_max_scratch_bytes(void);
int pkv_decode_attn_noalloc(const pkv_pool* pool, int32_t layer, const void* q,
                            int32_t num_q_heads, const pkv_page_table* table,
                            const int32_t* table_idx, const int32_t* seq_lens, int32_t batch,
                            float scale, void* out, int32_t* dev_err, pkv_stream_t stream);

/*
 * decode_attn_cascade -- decode_attn for batches whose requests share
 * radix-cached prefixes [P5 §1.4: requests with a common prefix point their
 * table rows at the same slots; §1.2: decode is memory bound].
 *
 *   The result is decode_attn's: out[r][h] = attention of q[r][h] over the
 *   first seq_lens[r] tokens of row table_idx[r].  The requests form
 *   num_groups contiguous groups, group g = requests group_offsets[g] ..
 *   group_offsets[g+1] - 1, whose first group_prefix_lens[g] context tokens
 *   are the same slots (the caller's promise: the call reads them from the
 *   row of the group's first request only).
 *
 * The shared prefix is attended once per group with all members' query rows
 * stacked on the tcgen05 tensor cores (its K/V are read once per group, not
 * once per request); each request's own suffix goes through the split-KV
 * decode kernel; the partial results are merged by their (max, sum) pairs.
 * This is not on the pages; it is the reuse their prefix sharing allows.
 * When the prefix pass is small (about 43% of the SMs' worth of CTAs or
 * less), it runs on a library-owned auxiliary stream beside the suffix pass,
 * forked from and joined back to `stream` with events, so the call stays
 * ordered on `stream` as a whole.  The auxiliary stream and its two events
 * are created once per device, on the first call made outside stream
 * capture; calls from several host threads are serialised around them.
 *
 * group_offsets: device int32 [num_groups + 1], 0 = first <= ... <= last =
 *   batch.  group_prefix_lens: device int32 [num_groups], each 0 <= p_g <=
 *   min over members of seq_lens and <= max_prefix_len (host int64, sizes
 *   the prefix pass and the workspace; <= table cols).  A violation sets
 *   PKV_DEV_ERR_BAD_LENGTH and the affected results are unspecified but
 *   finite.
 * workspace: pkv_decode_cascade_workspace_bytes(batch, num_q_heads,
 *   max_prefix_len) bytes, 16-byte aligned.
 * bf16 and FP8 pools (PKV_ERR_UNSUPPORTED for fp32); other limits as
 * decode_attn, with num_q_heads/num_kv_heads at most 8.
 */
size_t pkv_decode_cascade_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                          int64_t max_prefix_len);
int pkv_decode_attn_cascade(const pkv_pool* pool, int32_t layer, const void* q,
                            int32_t num_q_heads, const pkv_page_table* table,
                            const int32_t* table_idx, const int32_t* seq_lens, int32_t batch,
                            const int32_t* group_offsets, const int32_t* group_prefix_lens,
                            int32_t num_groups, int64_t max_prefix_len, float scale, void* out,
                            void* workspace, size_t workspace_bytes, int32_t* dev_err,
                            pkv_stream_t stream);

/*
 * extend_attn [P4 chunked prefill: every chunk of a request uses the same
 * table row and reuses the KV of the chunks before it; P5 §4.2.3: a request
 * has cached_len (its prefix, possibly radix-shared) and extend_len =
 * device_len - cached_len new tokens; §1.4: requests sharing a prefix point
 * their table rows at the same slots; §1.2: prefill is compute bound].
 *
 *   For request r with p = prefix_lens[r], e = extend_lens[r], query row
 *   i < e sits at position p + i and attends causally to keys 0 .. p + i:
 *   out[q_offsets[r] + i][h][:] = sum_{j <= p+i} softmax_j(scale * q[..][h]
 *   . K_r[j][h/G]) V_r[j][h/G].  The chunk's own K/V must already be in the
 *   pool (store_kv first, as the pages do).
 *
 * q, out: device [total_q][num_q_heads][head_dim] contiguous, pool dtype.
 * prefix_lens, extend_lens: device int32 [batch]; q_offsets: device int32
 *   [batch+1], q_offsets[0] = 0, q_offsets[r+1] = q_offsets[r] + extend_lens[r],
 *   q_offsets[batch] = total_q.
 * max_extend_len: host int, an upper bound on every extend_lens[r] (used to
 *   size the launch; rows beyond it are not computed and set
 *   PKV_DEV_ERR_BAD_LENGTH).
 * workspace: pkv_extend_workspace_bytes(...) bytes (currently 0 for bf16).
 * The bf16 path runs QK^T and PV on the tcgen05 tensor cores with TMEM
 * accumulators; the fp32 check build uses CUDA cores.  Same support limits
 * as decode_attn.
 */
size_t pkv_extend_workspace_bytes(int32_t batch, int32_t num_q_heads, int64_t total_q);
int pkv_extend_attn(const pkv_pool* pool, int32_t layer, const void* q, int32_t num_q_heads,
                    const pkv_page_table* table, const int32_t* table_idx,
                    const int32_t* prefix_lens, const int32_t* extend_lens,
                    const int32_t* q_offsets, int32_t batch, int64_t total_q,
                    int32_t max_extend_len, float scale, void* out, void* workspace,
                    size_t workspace_bytes, int32_t* dev_err, pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
