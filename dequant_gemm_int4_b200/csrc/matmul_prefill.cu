// Tensor-core (tcgen05) dequantizing matmul for large M, sm_100a.
// (Kernel under construction: no shape is accepted yet.)
#include "common.cuh"
#include "internal.h"

namespace int4lib {

bool prefill_supported(DType, int64_t, int, int64_t, int64_t, const void*, const uint8_t*) {
  return false;
}

cudaError_t launch_matmul_prefill(const void*, DType, const uint8_t*, const uint16_t*, int64_t, int,
                                  int64_t, int64_t, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace int4lib
