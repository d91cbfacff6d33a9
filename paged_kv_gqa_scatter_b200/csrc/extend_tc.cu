// Placeholder: routes bf16 extend to the CUDA-core kernel until the tensor-core kernel lands.
#include "launch.h"

namespace pkv {

cudaError_t launch_extend_tc(const PoolView& pool, const TableView& t, const void* q,
                             int32_t num_q_heads, const int32_t* table_idx,
                             const int32_t* prefix_lens, const int32_t* extend_lens,
                             const int32_t* q_offsets, int32_t batch, int64_t total_q, int32_t max_extend,
                             float scale, void* out, int32_t* err, cudaStream_t s) {
  return launch_extend_simt(pool, t, q, num_q_heads, table_idx, prefix_lens, extend_lens,
                            q_offsets, batch, total_q, max_extend, scale, out, err, s);
}

}  // namespace pkv
