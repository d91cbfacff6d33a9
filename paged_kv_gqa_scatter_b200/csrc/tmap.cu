// Driver entry point of cuTensorMapEncodeTiled, looked up once through the
// runtime (the library does not link libcuda directly).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "launch.h"

namespace pkv {

void* tensor_map_encode_fn() {
  static void* fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = ptr;
  }
  return fn;
}

}  // namespace pkv
