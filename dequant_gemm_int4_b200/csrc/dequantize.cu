// Dequantization of packed 4-bit weights to bf16, fp16 or fp32 (sm_100a).
//
// w_hat[n, k] = q[n, k] * s[n, k / group] for the symmetric scheme of the
// page "Implement INT4 group quantization, nibble packing and a dequantizing
// matmul" (q the two's-complement nibble, element 2j in the low nibble of
// byte j), and w_hat = (q - z[n, g]) * s[n, g] for the asymmetric scheme of
// "Build a Blockwise INT4 Inference Engine", step 2 (q the unsigned nibble,
// z the group's zero point), laid out the same way.  The product is exact in
// fp32 (a 4- or 5-bit integer times an fp16 scale) and rounded once, to
// nearest even, into the output type.
//
// HBM-bound: read 0.5 byte per weight (plus the group's scale), write 2 or 4.
// On rows whose length and group are multiples of 16 (and aligned buffers)
// each thread takes 16 weights of one row: one 8-byte load of nibbles, one
// scale, two or four 16-byte stores.  Other shapes take a byte-per-thread
// kernel.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace int4lib {

namespace {

template <typename TO>
struct Out;
template <>
struct Out<float> {
  __device__ __forceinline__ static void store16(float* p, const float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<float4*>(p)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  __device__ __forceinline__ static void store1(float* p, float v) { *p = v; }
};
template <>
struct Out<__nv_bfloat16> {
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // each rounded to nearest even
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  __device__ __forceinline__ static void store16(__nv_bfloat16* p, const float (&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack(v[2 * i], v[2 * i + 1]);
    reinterpret_cast<uint4*>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  __device__ __forceinline__ static void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <>
struct Out<__half> {
  __device__ __forceinline__ static uint32_t pack(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  __device__ __forceinline__ static void store16(__half* p, const float (&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack(v[2 * i], v[2 * i + 1]);
    reinterpret_cast<uint4*>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  __device__ __forceinline__ static void store1(__half* p, float v) { *p = __float2half_rn(v); }
};

// The integer weight of nibble `nib`: two's complement (symmetric) or the
// unsigned code minus the group's zero point (asymmetric).
template <bool ASYM>
__device__ __forceinline__ float weight_of(uint32_t nib, int zp) {
  if (ASYM) return static_cast<float>(static_cast<int>(nib) - zp);
  return static_cast<float>(static_cast<int32_t>(nib << 28) >> 28);
}

// Rows of K (a multiple of 16) weights, group a multiple of 16: chunk i is
// weights [16 c, 16 c + 16) of row r, i = r * (K / 16) + c.
template <typename TO, bool ASYM>
__global__ void __launch_bounds__(256) dequantize_flat_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ scales,
    const uint8_t* __restrict__ zeros, int64_t K, int group, int G, int64_t chunks,
    TO* __restrict__ out) {
  const int64_t cpr = K >> 4;  // chunks per row
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < chunks;
       i += stride) {
    const int64_t r = i / cpr;
    const int64_t c = i - r * cpr;
    const int g = static_cast<int>((c << 4) / group);
    const uint2 p = __ldg(reinterpret_cast<const uint2*>(packed) + i);
    const float s = f16_bits_to_float(__ldg(scales + r * G + g));
    const int zp = ASYM ? static_cast<int>(__ldg(zeros + r * G + g)) : 0;
    const uint32_t w[2] = {p.x, p.y};
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * h + j] = weight_of<ASYM>((w[h] >> (4 * j)) & 0xFu, zp) * s;
    Out<TO>::store16(out + (i << 4), v);
  }
}

// Any K, group and alignment: one packed byte (two weights) per thread.
template <typename TO, bool ASYM>
__global__ void __launch_bounds__(256) dequantize_any_kernel(
    const uint8_t* __restrict__ packed, const uint16_t* __restrict__ scales,
    const uint8_t* __restrict__ zeros, int64_t K, int group, int G, int64_t N,
    TO* __restrict__ out) {
  const int64_t Kp = (K + 1) >> 1;
  const int64_t total = N * Kp;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t r = i / Kp;
    const int64_t j = i - r * Kp;
    const uint32_t b = __ldg(packed + i);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t k = 2 * j + h;
      if (k >= K) break;  // the pad nibble of an odd K
      const int g = static_cast<int>(k / group);
      const float s = f16_bits_to_float(__ldg(scales + r * G + g));
      const int zp = ASYM ? static_cast<int>(__ldg(zeros + r * G + g)) : 0;
      Out<TO>::store1(out + r * K + k, weight_of<ASYM>((b >> (4 * h)) & 0xFu, zp) * s);
    }
  }
}

template <typename TO, bool ASYM>
cudaError_t launch_typed(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                         int64_t K, int group, int64_t N, TO* out, cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const bool flat = K % 16 == 0 && group % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(packed) % 8 == 0 &&
                    reinterpret_cast<uintptr_t>(out) % 16 == 0;
  if (flat) {
    const int64_t chunks = N * (K / 16);
    const int grid = resident_grid(dequantize_flat_kernel<TO, ASYM>, (chunks + 255) / 256);
    dequantize_flat_kernel<TO, ASYM><<<grid, 256, 0, stream>>>(packed, scales, zeros, K, group, G,
                                                              chunks, out);
  } else {
    const int64_t bytes = N * ((K + 1) / 2);
    const int grid = resident_grid(dequantize_any_kernel<TO, ASYM>, (bytes + 255) / 256);
    dequantize_any_kernel<TO, ASYM><<<grid, 256, 0, stream>>>(packed, scales, zeros, K, group, G,
                                                             N, out);
  }
  return cudaGetLastError();
}

template <bool ASYM>
cudaError_t launch_any(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                       int64_t K, int group, int64_t N, void* out, DType ot, cudaStream_t stream) {
  switch (ot) {
    case DType::F32:
      return launch_typed<float, ASYM>(packed, scales, zeros, K, group, N, static_cast<float*>(out), stream);
    case DType::BF16:
      return launch_typed<__nv_bfloat16, ASYM>(packed, scales, zeros, K, group, N,
                                               static_cast<__nv_bfloat16*>(out), stream);
    default:
      return launch_typed<__half, ASYM>(packed, scales, zeros, K, group, N, static_cast<__half*>(out),
                                        stream);
  }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                              int64_t K, int group, int64_t N, void* out, DType ot,
                              cudaStream_t stream) {
  if (zeros != nullptr) return launch_any<true>(packed, scales, zeros, K, group, N, out, ot, stream);
  return launch_any<false>(packed, scales, nullptr, K, group, N, out, ot, stream);
}

}  // namespace int4lib
