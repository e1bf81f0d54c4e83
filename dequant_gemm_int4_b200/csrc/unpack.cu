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

// Any K and alignment: a lane takes NB packed bytes (2 NB outputs), a warp a
// window of 64 NB outputs of one row.  A lane takes its aligned NB-byte
// chunk of the packed byte range, the next lane's chunk by shuffle,
// funnel-shifts by the row's byte offset, expands the nibbles and writes
// them with aligned word stores (store_segment).
#ifndef INT4_UNPACK_ANY_BYTES
#define INT4_UNPACK_ANY_BYTES 8
#endif
// packed bytes per lane: 8 measured faster than 16 (2.1 against 1.2 TB/s on
// W [8192, 28673]), whose eight clipped word stores per lane cost more than
// the halved window count saves.
constexpr int kUnpackAnyBytes = INT4_UNPACK_ANY_BYTES;

template <int NB>
__device__ __forceinline__ void load_packed_chunk(const uint8_t* base, int64_t c, int64_t nbytes,
                                                  uint32_t (&w)[NB / 4]) {
  if (NB == 8) {
    const uint2 v = load_chunk8(base, c, nbytes);
    w[0] = v.x;
    w[1] = v.y;
  } else {
    const uint4 v = load_chunk16(base, c, nbytes);
    w[0] = v.x;
    w[1] = v.y;
    w[NB / 4 > 2 ? 2 : 0] = v.z;
    w[NB / 4 > 3 ? 3 : 0] = v.w;
  }
}

template <int NB>
__global__ void __launch_bounds__(256) unpack_any_kernel(const uint8_t* __restrict__ pbase,
                                                        int64_t pshift, int64_t pbytes, int64_t K,
                                                        int64_t windows_per_row, int64_t total_windows,
                                                        uint8_t* __restrict__ obase, int64_t oshift) {
  static_assert(NB == 8 || NB == 16, "8- or 16-byte chunks");
  constexpr int NW = NB / 4;     // packed words per lane
  constexpr int WOUT = 64 * NB;  // outputs per window
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t per = (total_windows + nwarps - 1) / nwarps;
  int64_t wi = warp * per;
  const int64_t wend = (wi + per < total_windows) ? wi + per : total_windows;
  if (wi >= wend) return;
  const int64_t Kp = (K + 1) >> 1;
  int64_t row = wi / windows_per_row;
  int64_t col = wi - row * windows_per_row;

  // The next window's chunk is loaded while the current one is expanded.
  auto fetch = [&](int64_t r, int64_t cl, uint32_t (&own)[NW], uint32_t (&extra)[NW]) {
    const int64_t c = (pshift + r * Kp + cl * (32 * NB) + lane * NB) / NB;
    load_packed_chunk<NB>(pbase, c, pbytes, own);
    if (lane == 31) {
      load_packed_chunk<NB>(pbase, c + 1, pbytes, extra);
    } else {
#pragma unroll
      for (int j = 0; j < NW; ++j) extra[j] = 0u;
    }
  };
  uint32_t own[NW], extra[NW];
  fetch(row, col, own, extra);
  for (; wi < wend;) {
    uint32_t win[2 * NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) win[j] = own[j];
    uint32_t cur_extra[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) cur_extra[j] = extra[j];
    const int boff = static_cast<int>((pshift + row * Kp + col * (32 * NB) + lane * NB) & (NB - 1));
    const int64_t crow = row, ccol = col;
    if (++col == windows_per_row) {
      col = 0;
      ++row;
    }
    if (++wi < wend) fetch(row, col, own, extra);
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const uint32_t nx = __shfl_down_sync(0xffffffffu, win[j], 1);
      win[NW + j] = (lane == 31) ? cur_extra[j] : nx;
    }
    uint32_t bw[NW];
    byte_shift_words<2 * NW, NW>(win, boff, bw);
    uint32_t o[2 * NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const uint2 e = expand_word(bw[j]);
      o[2 * j] = e.x;
      o[2 * j + 1] = e.y;
    }
    const int64_t rowo = oshift + crow * K;
    const int64_t f0 = rowo + ccol * WOUT;
    const int64_t hi = (f0 + WOUT < rowo + K) ? f0 + WOUT : rowo + K;
    store_segment<2 * NW>(obase, f0, f0, hi, o, lane);
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
  constexpr int NB = kUnpackAnyBytes;
  const uintptr_t pa = reinterpret_cast<uintptr_t>(packed);
  const uint8_t* pbase = reinterpret_cast<const uint8_t*>(pa & ~static_cast<uintptr_t>(NB - 1));
  const int64_t pshift = static_cast<int64_t>(pa & (NB - 1));
  const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
  uint8_t* obase = reinterpret_cast<uint8_t*>(oa & ~static_cast<uintptr_t>(3));
  const int64_t oshift = static_cast<int64_t>(oa & 3);
  const int64_t wpr = (K + 64 * NB - 1) / (64 * NB);
  const int64_t total = N * wpr;
  const int grid = resident_grid(unpack_any_kernel<NB>, (total + 31) / 32);
  unpack_any_kernel<NB><<<grid, 256, 0, stream>>>(
      pbase, pshift, pshift + N * ((K + 1) / 2), K, wpr, total, obase, oshift);
  return cudaGetLastError();
}

}  // namespace int4lib
