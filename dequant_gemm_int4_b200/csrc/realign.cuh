// Warp-cooperative access to byte ranges that start at any alignment.
//
// Rows of an odd-K matrix start at arbitrary byte offsets (bf16 rows at 2K
// bytes, packed rows at ceil(K/2) bytes), so a warp that walks a row cannot
// use aligned vector loads and stores directly.  These helpers keep every
// global access aligned: a lane loads its own aligned chunk, receives the next
// lane's chunk with a shuffle, and funnel-shifts by the (warp-uniform) byte
// offset; stores write aligned 32-bit words and fall back to single bytes
// only for words that straddle the clip range (segment ends, row ends).
#pragma once

#include <stdint.h>

namespace int4lib {

// Word j of the concatenation (w[0..n), ...) shifted right by `boff` bytes
// (0 <= boff < 4 * (n - NOUT)), for NOUT output words.
template <int NIN, int NOUT>
__device__ __forceinline__ void byte_shift_words(const uint32_t (&w)[NIN], int boff,
                                                 uint32_t (&out)[NOUT]) {
  static_assert(NIN > NOUT, "need at least one extra word");
  const int q = boff >> 2;
  const uint32_t r = static_cast<uint32_t>(boff & 3) * 8u;
  uint32_t t[NIN];
#pragma unroll
  for (int i = 0; i < NIN; ++i) t[i] = w[i];
  // Word shift by q in binary steps (q < NIN - NOUT).
#pragma unroll
  for (int step = 1; step < NIN - NOUT + 1; step <<= 1) {
    if (q & step) {
#pragma unroll
      for (int i = 0; i + step < NIN; ++i) t[i] = t[i + step];
    }
  }
#pragma unroll
  for (int j = 0; j < NOUT; ++j) out[j] = __funnelshift_r(t[j], t[j + 1], r);
}

// Loads the aligned 16-byte chunk `c` of `base` (16-byte aligned); bytes at or
// past `nbytes` read as zero and are never touched in memory.
__device__ __forceinline__ uint4 load_chunk16(const uint8_t* base, int64_t c, int64_t nbytes) {
  const int64_t b0 = c * 16;
  if (b0 + 16 <= nbytes) return __ldg(reinterpret_cast<const uint4*>(base) + c);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int i = 0; i < 16; ++i)
    if (b0 + i < nbytes) w[i >> 2] |= static_cast<uint32_t>(__ldg(base + b0 + i)) << (8 * (i & 3));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Loads the aligned 8-byte chunk `c` of `base` (8-byte aligned), zero past `nbytes`.
__device__ __forceinline__ uint2 load_chunk8(const uint8_t* base, int64_t c, int64_t nbytes) {
  const int64_t b0 = c * 8;
  if (b0 + 8 <= nbytes) return __ldg(reinterpret_cast<const uint2*>(base) + c);
  uint32_t w[2] = {0u, 0u};
  for (int i = 0; i < 8; ++i)
    if (b0 + i < nbytes) w[i >> 2] |= static_cast<uint32_t>(__ldg(base + b0 + i)) << (8 * (i & 3));
  return make_uint2(w[0], w[1]);
}

// Writes the 4 bytes of `v` to base[pos .. pos+4) (pos 4-byte aligned in the
// address space of `base`), clipped to [lo, hi).
__device__ __forceinline__ void store_word_clipped(uint8_t* base, int64_t pos, uint32_t v, int64_t lo,
                                                   int64_t hi) {
  if (pos >= lo && pos + 4 <= hi) {
    *reinterpret_cast<uint32_t*>(base + pos) = v;
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (pos + i >= lo && pos + i < hi) base[pos + i] = static_cast<uint8_t>(v >> (8 * i));
}

// The warp holds a contiguous byte segment: lane l holds bytes
// [f0 + 4*NW*l, f0 + 4*NW*(l+1)) as NW little-endian words.  Writes the part of
// it inside [lo, hi) to `base` (4-byte aligned) with aligned word stores.
template <int NW>
__device__ __forceinline__ void store_segment(uint8_t* base, int64_t f0, int64_t lo, int64_t hi,
                                              const uint32_t (&w)[NW], int lane) {
  const int off = static_cast<int>(f0 & 3);
  const int64_t b = f0 - off + static_cast<int64_t>(4 * NW) * lane;  // aligned word below lane start
  const uint32_t nxt = __shfl_down_sync(0xffffffffu, w[0], 1);
  uint32_t e[NW + 1];
#pragma unroll
  for (int j = 0; j < NW; ++j) e[j] = w[j];
  e[NW] = nxt;
  const uint32_t sh = static_cast<uint32_t>(4 - off) * 8u;  // 8..32 bits
  // Word at b: only lane 0 writes it (its low `off` bytes belong to the
  // previous segment); other lanes' word at b is written by the lane before.
  if (lane == 0) store_word_clipped(base, b, w[0] << (8 * off), lo, hi);
#pragma unroll
  for (int j = 0; j < NW; ++j)
    store_word_clipped(base, b + 4 + 4 * j, __funnelshift_rc(e[j], e[j + 1], sh), lo, hi);
}

}  // namespace int4lib
