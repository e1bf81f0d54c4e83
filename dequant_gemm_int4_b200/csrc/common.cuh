// Device helpers shared by the kernels of the INT4 library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace int4lib {

// Element widening.  bf16 and fp16 widen to fp32 exactly.
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}
__device__ __forceinline__ float f16_bits_to_float(uint32_t bits16) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)));
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  __device__ __forceinline__ static float load(const float* p) { return __ldg(p); }
};
template <>
struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
    return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p)));
  }
};
template <>
struct Elem<__half> {
  __device__ __forceinline__ static float load(const __half* p) {
    return f16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p)));
  }
};

// What the matmul kernels do to an output before storing it: add the output
// column's bias (fp32 [N], optional), then ReLU (max(v, 0), NaN kept), as the
// linear layer of the page "Build a Blockwise INT4 Inference Engine", steps 3
// and 4 (x @ W_dq^T + bias, then ReLU).
struct Epilogue {
  const float* bias = nullptr;
  int relu = 0;
  __device__ __forceinline__ float apply(float v, int64_t n) const {
    if (bias != nullptr) v += __ldg(bias + n);
    if (relu != 0 && v < 0.0f) v = 0.0f;
    return v;
  }
};

// Kernels whose bounded waits give up OR a bit into the library's
// device-side status word; its address comes from status_word().
__device__ __forceinline__ void report_status(uint32_t* status, uint32_t bit) {
  atomicOr(status, bit);
}

}  // namespace int4lib
