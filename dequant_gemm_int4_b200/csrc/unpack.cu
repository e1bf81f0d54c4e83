// Nibble unpacking with sign extension (sm_100a).
//
// Follows unpack_int4(packed, K) -> int8 [N, K] of the page "Implement INT4
// group quantization, nibble packing and a dequantizing matmul" (problem
// statement): element 2j is the low nibble of byte j, element 2j+1 the high
// nibble, each a 4-bit two's-complement value.
//
// HBM-bound (read N*ceil(K/2) bytes, write N*K bytes).  For even K the packed
// rows are contiguous nibble streams, so the whole matrix is one flat
// elementwise map: each thread turns 8 packed bytes (one 8-byte load) into 16
// int8 outputs (one 16-byte store).
#include "common.cuh"
#include "internal.h"

namespace int4lib {

namespace {

// 4 packed bytes -> 8 sign-extended int8 values (two 32-bit words).
__device__ __forceinline__ uint2 expand_word(uint32_t w) {
  const uint32_t lo = w & 0x0F0F0F0Fu;
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
  uint32_t a = __byte_perm(lo, hi, 0x5140);  // lo.b0 hi.b0 lo.b1 hi.b1
  uint32_t b = __byte_perm(lo, hi, 0x7362);  // lo.b2 hi.b2 lo.b3 hi.b3
  // Sign extension per byte: a nibble with bit 3 set gets 0xF0 in its top half.
  a |= (a & 0x08080808u) * 0x1Eu;
  b |= (b & 0x08080808u) * 0x1Eu;
  return make_uint2(a, b);
}

__device__ __forceinline__ int8_t sext4(uint32_t nib) {
  return static_cast<int8_t>(static_cast<int32_t>(nib << 28) >> 28);
}

// Even K, packed 8-byte aligned and out 16-byte aligned: flat map.
__global__ void __launch_bounds__(256) unpack_flat_kernel(const uint8_t* __restrict__ packed,
                                                         int64_t total_bytes,
                                                         int8_t* __restrict__ out) {
  const int64_t nvec = total_bytes >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += stride) {
    const uint2 p = __ldg(reinterpret_cast<const uint2*>(packed) + i);
    const uint2 a = expand_word(p.x);
    const uint2 b = expand_word(p.y);
    reinterpret_cast<uint4*>(out)[i] = make_uint4(a.x, a.y, b.x, b.y);
  }
  // Tail bytes (total_bytes not a multiple of 8): one thread.
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t j = nvec << 3; j < total_bytes; ++j) {
      const uint32_t byte = packed[j];
      out[2 * j] = sext4(byte & 0xFu);
      out[2 * j + 1] = sext4(byte >> 4);
    }
  }
}

// General K and alignment: one thread per output element.
__global__ void __launch_bounds__(256) unpack_general_kernel(const uint8_t* __restrict__ packed,
                                                            int64_t N, int64_t K,
                                                            int8_t* __restrict__ out) {
  const int64_t Kp = (K + 1) >> 1;
  const int64_t total = N * K;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += stride) {
    const int64_t n = e / K;
    const int64_t k = e - n * K;
    const uint32_t byte = __ldg(packed + n * Kp + (k >> 1));
    out[e] = sext4((k & 1) ? (byte >> 4) : (byte & 0xFu));
  }
}

}  // namespace

cudaError_t launch_unpack(const uint8_t* packed, int64_t K, int64_t N, int8_t* out,
                          cudaStream_t stream) {
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (K % 2 == 0 && reinterpret_cast<uintptr_t>(packed) % 8 == 0 &&
      reinterpret_cast<uintptr_t>(out) % 16 == 0) {
    const int64_t total = N * (K / 2);
    int64_t grid = ((total >> 3) + 255) / 256;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    unpack_flat_kernel<<<static_cast<int>(grid), 256, 0, stream>>>(packed, total, out);
    return cudaGetLastError();
  }
  int64_t grid = (N * K + 255) / 256;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  unpack_general_kernel<<<static_cast<int>(grid), 256, 0, stream>>>(packed, N, K, out);
  return cudaGetLastError();
}

}  // namespace int4lib
