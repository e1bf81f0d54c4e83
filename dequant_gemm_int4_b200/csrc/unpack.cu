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
#include "realign.cuh"

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

// Any K and alignment, row by row (blockIdx.y walks the rows): output row r
// is the byte range [o_r, o_r + K) with o_r = oshift + r K from the 16-byte
// aligned `obase`.  A thread writes one aligned 16-byte chunk that lies
// inside the row: its outputs are nibbles col .. col + 15 of packed row r;
// the thread loads the two aligned 8-byte words around them (its neighbours
// read the same words, from L1), shifts the pair by the byte and nibble
// offset, expands the 16 nibbles and stores them with one 16-byte store.  The
// row's bytes before its first and after its last whole chunk (fewer than 16
// at each end) are written byte by byte, so neighbouring rows never write the
// same byte.
__device__ __forceinline__ uint8_t unpack_byte(const uint8_t* pbase, int64_t prow, int64_t col) {
  const uint32_t byte = pbase[prow + (col >> 1)];
  return static_cast<uint8_t>(sext4((col & 1) ? (byte >> 4) : (byte & 0xFu)));
}

__global__ void __launch_bounds__(256) unpack_rows_kernel(
    const uint8_t* __restrict__ pbase, int64_t pshift, int64_t pbytes, int64_t N, int64_t K,
    uint8_t* __restrict__ obase, int64_t oshift) {
  const int64_t Kp = (K + 1) >> 1;
  for (int64_t r = blockIdx.y; r < N; r += gridDim.y) {
    const int64_t o0 = oshift + r * K;      // row start, bytes from obase
    const int64_t cA = (o0 + 15) >> 4;      // first whole chunk
    const int64_t cB = (o0 + K) >> 4;       // one past the last whole chunk
    const int64_t prow = pshift + r * Kp;   // packed row start, bytes from pbase
    for (int64_t c = cA + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < cB;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t col = 16 * c - o0;
      const int64_t B = prow + (col >> 1);
      const uint32_t sh = static_cast<uint32_t>(B & 7) * 8u + static_cast<uint32_t>(col & 1) * 4u;
      const uint2 l = load_chunk8(pbase, B >> 3, pbytes);
      const uint2 h = load_chunk8(pbase, (B >> 3) + 1, pbytes);
      const uint64_t lo = (static_cast<uint64_t>(l.y) << 32) | l.x;
      const uint64_t hi = (static_cast<uint64_t>(h.y) << 32) | h.x;
      const uint64_t v = sh == 0u ? lo : (lo >> sh) | (hi << (64u - sh));
      const uint2 x = expand_word(static_cast<uint32_t>(v));
      const uint2 y = expand_word(static_cast<uint32_t>(v >> 32));
      reinterpret_cast<uint4*>(obase)[c] = make_uint4(x.x, x.y, y.x, y.y);
    }
    if (blockIdx.x == 0 && threadIdx.x < 32) {
      // The ends: [o0, 16 cA) and [16 cB, o0 + K), or the whole row when it
      // holds no whole chunk.
      const int64_t head_end = (cA < cB) ? 16 * cA - o0 : K;
      const int64_t tail_beg = (cA < cB) ? 16 * cB - o0 : K;
      const int i = threadIdx.x;
      for (int64_t col = i; col < head_end; col += 32) obase[o0 + col] = unpack_byte(pbase, prow, col);
      for (int64_t col = tail_beg + i; col < K; col += 32) obase[o0 + col] = unpack_byte(pbase, prow, col);
    }
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
  const uintptr_t pa = reinterpret_cast<uintptr_t>(packed);
  const uint8_t* pbase = reinterpret_cast<const uint8_t*>(pa & ~static_cast<uintptr_t>(7));
  const int64_t pshift = static_cast<int64_t>(pa & 7);
  const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
  uint8_t* obase = reinterpret_cast<uint8_t*>(oa & ~static_cast<uintptr_t>(15));
  const int64_t oshift = static_cast<int64_t>(oa & 15);
  // Blocks per row cover its whole chunks (K / 16 + 1 at most); the rows go
  // to blockIdx.y, up to the grid's limit, then stride.
  const int64_t bx = (K / 16 + 1 + 255) / 256;
  const int64_t by = N < 65535 ? N : 65535;
  unpack_rows_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(by)), 256, 0, stream>>>(
      pbase, pshift, pshift + N * ((K + 1) / 2), N, K, obase, oshift);
  return cudaGetLastError();
}

}  // namespace int4lib
