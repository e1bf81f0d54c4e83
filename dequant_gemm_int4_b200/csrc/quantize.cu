// Group-wise INT4 quantization and nibble packing (sm_100a).
//
// Follows the quantize_int4 function of the page "Implement INT4 group
// quantization, nibble packing and a dequantizing matmul" (problem
// statement): per row and per K-group, scale = absmax / 7 stored as fp16,
// q = round(w / scale) clamped to [-8, 7], two's-complement nibbles with
// element 2j in the low nibble of byte j, a zero pad nibble for odd K and
// scale 0 for an all-zero group.  Rounding convention: fp32 IEEE division
// absmax / 7, then round-to-nearest-even to fp16; q = rint_half_even of the
// IEEE fp32 quotient w / float(scale).
//
// HBM-bound: every weight is read once (fp32/bf16/fp16) and the packed codes
// and scales written once.  The fast kernel gives each warp a window of 32
// consecutive 8-element chunks of one row (one 16-byte load per lane for
// 16-bit weights), reduces the group absmax with warp shuffles across the
// group/8 lanes of each group, and stores 4 packed bytes per lane.
#include "common.cuh"
#include "internal.h"
#include "realign.cuh"

namespace int4lib {

namespace {

struct ScaleInfo {
  uint32_t bits;  // fp16 bit pattern of the scale
  float sf;       // the scale widened to fp32
  float r;        // approximately 1 / sf (0 when sf is 0 or +inf)
};

// fp32(m / 7), correctly rounded, for finite m >= 0.  Division by a constant
// with one residual correction (Markstein's method for a known divisor):
// q0 = m * c with c = fp32(1/7), the residual e = m - 7 q0 is exact by FMA,
// and q1 = q0 + e * c is the correctly rounded quotient.  The test suite
// checks it against the IEEE division for every fp32 mantissa over the
// normal exponents whose behaviour differs, and over the whole subnormal
// range.
__device__ __forceinline__ float div7_rn(float m) {
  const float c = 0.142857149f;  // fp32 nearest to 1/7
  const float q0 = __fmul_rn(m, c);
  const float e = __fmaf_rn(-7.0f, q0, m);
  return __fmaf_rn(e, c, q0);
}

// Hardware reciprocal approximation (relative error about 2^-23); only the
// fast-path quotient uses it, which the certified check in code_fast covers.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ ScaleInfo scale_from_bits(uint32_t bits) {
  ScaleInfo si;
  si.bits = bits;
  si.sf = f16_bits_to_float(bits);
  si.r = (si.sf == 0.0f || bits == 0x7C00u) ? 0.0f : rcp_approx(si.sf);
  return si;
}

// s = fp16_RNE(fp32(m) / 7): the correctly rounded fp32 quotient, then RNE to fp16.
__device__ __forceinline__ ScaleInfo scale_from_absmax(float m) {
  const __half h = __float2half_rn(div7_rn(m));
  return scale_from_bits(__half_as_ushort(h));
}

// The 4-bit code of v: clamp(rint(fp32(v / sf)), -8, 7), 0 when sf == 0,
// with the IEEE division (used on the rare path and by the general kernels).
__device__ __forceinline__ uint32_t code_exact(float v, const ScaleInfo& si) {
  if (si.sf == 0.0f) return 0u;
  float rt = rintf(__fdiv_rn(v, si.sf));
  rt = fminf(fmaxf(rt, -8.0f), 7.0f);
  return static_cast<uint32_t>(static_cast<int>(rt)) & 0xFu;
}

// Fast path of the same code.  The quotient is approximated as t = v * r
// with r within 2^-22 (relative) of 1/sf.  With x the exact quotient,
// |t - x| <= |x| * 2^-21, and the correctly rounded fp32(x) lies within
// another half ulp of x, so for |x| < 16 both differ from t by less than
// 2^-16.  rint(fp32(x)) can only differ from rint(t) if a half-integer lies
// within that distance of t; `near` is then set and the caller recomputes
// with the IEEE division.  Clamping before rounding is the same as after
// (the bounds are integers), and a clamped t is far from every half-integer
// that can change the result (+-7.5 and beyond never do).  Rounding uses the
// exact magic-number addition t + 1.5 * 2^23, whose fp32 result holds rint(t)
// (ties to even) in its low mantissa bits, so the nibble is read from the bit
// pattern and no conversion instruction is needed.
__device__ __forceinline__ uint32_t code_fast(float v, float r, bool& near) {
  const float t = fminf(fmaxf(__fmul_rn(v, r), -8.0f), 7.0f);
  const float yv = __fadd_rn(t, 12582912.0f);
  const float d = __fsub_rn(t, __fsub_rn(yv, 12582912.0f));
  near = near || (fabsf(d) >= 0.5f - 0x1p-15f);
  return __float_as_uint(yv) & 0xFu;
}

// Eight codes of one lane for a normal fp16 scale (2^-14 <= s < +inf), packed
// low nibble first.  Then |v / s| <= 7 / (1 - 2^-11) < 7.5, so no clamp is
// needed, and t = v * r stays within 2^-16 of the exact quotient (see
// code_fast).  Returns false if some quotient lies too close to a
// half-integer, in which case the caller recomputes exactly.
__device__ __forceinline__ bool codes8_normal(const float (&v)[8], float r, uint32_t& word) {
  float dmax = 0.0f;
  uint32_t nib[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = __fmul_rn(v[i], r);
    const float yv = __fadd_rn(t, 12582912.0f);
    const float d = __fsub_rn(t, __fsub_rn(yv, 12582912.0f));
    dmax = fmaxf(dmax, fabsf(d));
    nib[i] = __float_as_uint(yv);
  }
  // Two nibbles per byte, four bytes per word.
  uint32_t b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t o;
    asm("lop3.b32 %0, %1, %2, %3, 0xb8;" : "=r"(o) : "r"(nib[2 * j + 1] << 4), "r"(0x0Fu), "r"(nib[2 * j]));
    b[j] = o;  // (hi << 4 & ~0x0F) | (lo & 0x0F): byte 0 holds both nibbles
  }
  word = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  return dmax < 0.5f - 0x1p-15f;
}

// Eight codes of one lane for 16-bit weights (bf16 or fp16) and a normal
// fp16 scale, packed low nibble first; exact with no check.  For such inputs
// a quotient v / s that is not itself a half-integer lies at least 2^-14
// away from every half-integer: 2v - (2k + 1)s is a multiple of the smaller
// of the two unit steps (of 2v and of s), and dividing that step by 2s leaves
// at least 2^-14 when |v / s| >= 1/8 (smaller quotients round to 0 anyway).
// fma(v, r, 192) rounds v * r (within 2^-19.5 of the quotient) to the 2^-16
// grid of [128, 256), which puts an exact tie exactly on k + 1/2 and leaves
// every other quotient on its own side of the nearest half-integer; adding
// 1.5 * 2^23 - 192 then rounds that grid value to an integer, ties to even,
// as rint does on the IEEE quotient.
__device__ __forceinline__ void codes8_snap(const float (&v)[8], float r, uint32_t& word) {
  // Two weights per instruction (packed fp32 FMA and add, each lane rounded
  // exactly as its scalar form).
  uint32_t nib[8];
  const float2 rr = make_float2(r, r);
  const float2 c192 = make_float2(192.0f, 192.0f);
  const float2 cmag = make_float2(12582720.0f, 12582720.0f);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 y1 = __ffma2_rn(make_float2(v[i], v[i + 1]), rr, c192);
    const float2 yv = __fadd2_rn(y1, cmag);
    nib[i] = __float_as_uint(yv.x);
    nib[i + 1] = __float_as_uint(yv.y);
  }
  uint32_t b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t o;
    asm("lop3.b32 %0, %1, %2, %3, 0xb8;" : "=r"(o) : "r"(nib[2 * j + 1] << 4), "r"(0x0Fu), "r"(nib[2 * j]));
    b[j] = o;
  }
  word = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
}

// Codes of eight weights of type T under a normal (or zero) scale: the
// checked fast path for fp32 weights, the snapped one for 16-bit weights.
template <typename T>
__device__ __forceinline__ bool codes8(const float (&v)[8], float r, uint32_t& word) {
  if (sizeof(T) == 2) {
    codes8_snap(v, r, word);
    return true;
  }
  return codes8_normal(v, r, word);
}

// The exact code, via the fast path and its check (general kernels).
__device__ __forceinline__ uint32_t code_of(float v, const ScaleInfo& si) {
  bool near = false;
  const uint32_t q = code_fast(v, si.r, near);
  return near ? code_exact(v, si) : q;
}

// Load 8 consecutive elements starting at p (16-byte aligned) as fp32.
template <typename T>
struct Load8;
template <>
struct Load8<float> {
  __device__ __forceinline__ static void run(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <>
struct Load8<__nv_bfloat16> {
  __device__ __forceinline__ static void run(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <>
struct Load8<__half> {
  __device__ __forceinline__ static void run(const __half* p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = f16_bits_to_float(w[i] & 0xFFFFu);
      v[2 * i + 1] = f16_bits_to_float(w[i] >> 16);
    }
  }
};

constexpr int kUnroll = 4;  // windows in flight per warp

// Fast path: K % 8 == 0, group = 8 * LPG with LPG a power of two <= 32,
// w 16-byte aligned, packed 4-byte aligned.  One warp window = 32 chunks of 8
// elements of one row.  Windows are numbered row-major over (row, window);
// each warp takes a contiguous range of them, so the row and window of the
// next one follow by increment (no division in the loop).
template <typename T, int LPG>
__global__ void __launch_bounds__(256) quantize_aligned_kernel(
    const T* __restrict__ w, int64_t K, int G, int64_t windows_per_row, int64_t total_windows,
    uint8_t* __restrict__ packed, uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t per = (total_windows + nwarps - 1) / nwarps;
  int64_t wbeg = warp * per;
  const int64_t wend = (wbeg + per < total_windows) ? wbeg + per : total_windows;
  if (wbeg >= wend) return;
  const int chunks_per_row = static_cast<int>(K >> 3);
  const int64_t Kp = K >> 1;
  int64_t row = wbeg / windows_per_row;
  int col = static_cast<int>(wbeg - row * windows_per_row);
  const int wpr = static_cast<int>(windows_per_row);

  for (; wbeg < wend; wbeg += kUnroll) {
    float v[kUnroll][8];
    int64_t rw[kUnroll];
    int ch[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      rw[u] = row;
      ch[u] = col * 32 + lane;
      valid[u] = (wbeg + u < wend) && (ch[u] < chunks_per_row);
      if (valid[u]) {
        Load8<T>::run(w + row * K + static_cast<int64_t>(ch[u]) * 8, v[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.0f;
      }
      if (++col == wpr) {
        col = 0;
        ++row;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[u][i]));
#pragma unroll
      for (int off = 1; off < LPG; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const ScaleInfo si = scale_from_absmax(m);
      // Normal scale (exponent field neither 0 nor all ones) or zero scale
      // (r == 0 makes every code 0) take the fast path; subnormal and
      // infinite scales (rare) go to the exact path.
      const uint32_t ex = si.bits & 0x7C00u;
      const bool simple = (ex != 0u && ex != 0x7C00u) || si.bits == 0u;
      uint32_t word;
      const bool ok = codes8<T>(v[u], si.r, word) && simple;
      if (!__all_sync(0xffffffffu, ok)) {
        if (!ok) {
          word = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) word |= code_exact(v[u][i], si) << (4 * i);
        }
      }
      if (valid[u]) {
        if ((lane & (LPG - 1)) == 0) scales[rw[u] * G + ch[u] / LPG] = static_cast<uint16_t>(si.bits);
        *reinterpret_cast<uint32_t*>(packed + rw[u] * Kp + static_cast<int64_t>(ch[u]) * 4) = word;
      }
    }
  }
}

// Wide fast path: K % 16 == 0, group = 16 * LPG (LPG a power of two <= 32),
// w 16-byte aligned, packed 8-byte aligned.  Each lane takes 16 consecutive
// elements per window (two 16-byte loads for 16-bit weights) and stores 8
// packed bytes, so the per-window work (scale, shuffles, addressing, stores)
// is spread over twice as many elements as in quantize_aligned_kernel.
template <typename T, int LPG>
__global__ void __launch_bounds__(256) quantize_wide_kernel(
    const T* __restrict__ w, int64_t K, int G, int64_t windows_per_row, int64_t total_windows,
    uint8_t* __restrict__ packed, uint16_t* __restrict__ scales) {
  constexpr int kU = 2;                                       // windows per step
  constexpr int kV = sizeof(T) == 4 ? 4 : 2;                  // 16-byte loads per lane per window
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t per = (total_windows + nwarps - 1) / nwarps;
  int64_t wbeg = warp * per;
  const int64_t wend = (wbeg + per < total_windows) ? wbeg + per : total_windows;
  if (wbeg >= wend) return;
  const int chunks_per_row = static_cast<int>(K >> 4);
  const int64_t Kp = K >> 1;
  int64_t row = wbeg / windows_per_row;
  int col = static_cast<int>(wbeg - row * windows_per_row);
  const int wpr = static_cast<int>(windows_per_row);

  // Raw 16-byte words of the next step are loaded while the current one is
  // quantized, so every warp keeps its next loads in flight.
  uint4 raw[kU][kV], nraw[kU][kV];
  int64_t rw[kU], nrw[kU];
  int ch[kU], nch[kU];
  bool valid[kU], nvalid[kU];
  auto fetch = [&](int64_t wb, uint4 (&r)[kU][kV], int64_t (&rr)[kU], int (&cc)[kU], bool (&vv)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      rr[u] = row;
      cc[u] = col * 32 + lane;
      vv[u] = (wb + u < wend) && (cc[u] < chunks_per_row);
      const uint4* p = reinterpret_cast<const uint4*>(w + row * K + static_cast<int64_t>(cc[u]) * 16);
#pragma unroll
      for (int q = 0; q < kV; ++q) r[u][q] = vv[u] ? __ldg(p + q) : make_uint4(0u, 0u, 0u, 0u);
      if (++col == wpr) {
        col = 0;
        ++row;
      }
    }
  };
  fetch(wbeg, nraw, nrw, nch, nvalid);
  for (; wbeg < wend; wbeg += kU) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      rw[u] = nrw[u];
      ch[u] = nch[u];
      valid[u] = nvalid[u];
#pragma unroll
      for (int q = 0; q < kV; ++q) raw[u][q] = nraw[u][q];
    }
    if (wbeg + kU < wend) fetch(wbeg + kU, nraw, nrw, nch, nvalid);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float v[2][8];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (sizeof(T) == 4) {
          const uint4 a = raw[u][2 * hh], bq = raw[u][2 * hh + 1];
          const uint32_t ws[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) v[hh][i] = __uint_as_float(ws[i]);
        } else {
          const uint4 a = raw[u][hh];
          const uint32_t ws[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (std::is_same<T, __nv_bfloat16>::value) {
              v[hh][2 * i] = __uint_as_float(ws[i] << 16);
              v[hh][2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
            } else {
              v[hh][2 * i] = f16_bits_to_float(ws[i] & 0xFFFFu);
              v[hh][2 * i + 1] = f16_bits_to_float(ws[i] >> 16);
            }
          }
        }
      }
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fmaxf(fabsf(v[0][i]), fabsf(v[1][i])));
#pragma unroll
      for (int off = 1; off < LPG; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const ScaleInfo si = scale_from_absmax(m);
      const uint32_t ex = si.bits & 0x7C00u;
      const bool simple = (ex != 0u && ex != 0x7C00u) || si.bits == 0u;
      uint32_t w0, w1;
      const bool ok0 = codes8<T>(v[0], si.r, w0);
      const bool ok1 = codes8<T>(v[1], si.r, w1);
      const bool ok = ok0 && ok1 && simple;
      if (!__all_sync(0xffffffffu, ok)) {
        if (!ok) {
          w0 = 0;
          w1 = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            w0 |= code_exact(v[0][i], si) << (4 * i);
            w1 |= code_exact(v[1][i], si) << (4 * i);
          }
        }
      }
      if (valid[u]) {
        if ((lane & (LPG - 1)) == 0) scales[rw[u] * G + ch[u] / LPG] = static_cast<uint16_t>(si.bits);
        *reinterpret_cast<uint2*>(packed + rw[u] * Kp + static_cast<int64_t>(ch[u]) * 8) =
            make_uint2(w0, w1);
      }
    }
  }
}

#ifndef INT4_QUANT_ANY_CHUNKS
#define INT4_QUANT_ANY_CHUNKS 4
#endif
constexpr int kAnyChunks16 = INT4_QUANT_ANY_CHUNKS;  // 16-byte chunks per lane, 16-bit weights

// Rows at any alignment (odd K, unaligned pointers), same groups as the fast
// path.  A lane takes EPL consecutive elements (NCH 16-byte chunks: 8 NCH for
// 16-bit weights, 8 for fp32), a warp a window of 32 EPL elements
// of one row.  The weights are read as aligned 16-byte chunks of the byte
// range that starts at `wbase` (16-byte aligned, w[0,0] at byte `wshift`): a
// lane loads its chunks, takes the next lane's first chunk by shuffle and
// funnel-shifts by the row's byte offset, which is the same for every lane of
// the window.  Packed bytes are written as aligned words with store_segment.
template <typename T, int LPG, int NCH>
__global__ void __launch_bounds__(256) quantize_any_kernel(
    const uint8_t* __restrict__ wbase, int64_t wshift, int64_t wbytes, int64_t K, int G,
    int64_t windows_per_row, int64_t total_windows, uint8_t* __restrict__ pbase, int64_t pshift,
    uint16_t* __restrict__ scales) {
  constexpr int ELT = static_cast<int>(sizeof(T));
  constexpr int EPL = NCH * 16 / ELT;  // elements per lane
  constexpr int WIN = 32 * EPL;        // elements per window
  constexpr int PW = EPL / 8;          // packed words per lane
  static_assert(EPL % 8 == 0, "whole 8-element code words per lane");
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

  // The next window's chunks are loaded while the current one is quantized.
  auto fetch = [&](int64_t r, int64_t cl, uint4 (&own)[NCH], uint4& extra) {
    const int64_t c0 = (wshift + (r * K + cl * WIN + lane * EPL) * ELT) >> 4;
#pragma unroll
    for (int q = 0; q < NCH; ++q) own[q] = load_chunk16(wbase, c0 + q, wbytes);
    extra = (lane == 31) ? load_chunk16(wbase, c0 + NCH, wbytes) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 own[NCH], extra;
  fetch(row, col, own, extra);
  for (; wi < wend;) {
    uint4 cur[NCH];
#pragma unroll
    for (int q = 0; q < NCH; ++q) cur[q] = own[q];
    const uint4 cur_extra = extra;
    const int64_t kl = col * WIN + lane * EPL;  // first element of this lane in the row
    const int64_t P = wshift + (row * K + kl) * ELT;
    const int boff = static_cast<int>(P & 15);
    const int64_t crow = row, ccol = col;
    if (++col == windows_per_row) {
      col = 0;
      ++row;
    }
    if (++wi < wend) fetch(row, col, own, extra);
    uint32_t win[4 * (NCH + 1)];
#pragma unroll
    for (int q = 0; q < NCH; ++q) {
      win[4 * q] = cur[q].x; win[4 * q + 1] = cur[q].y; win[4 * q + 2] = cur[q].z; win[4 * q + 3] = cur[q].w;
    }
    uint4 nx;
    nx.x = __shfl_down_sync(0xffffffffu, win[0], 1);
    nx.y = __shfl_down_sync(0xffffffffu, win[1], 1);
    nx.z = __shfl_down_sync(0xffffffffu, win[2], 1);
    nx.w = __shfl_down_sync(0xffffffffu, win[3], 1);
    if (lane == 31) nx = cur_extra;
    win[4 * NCH] = nx.x; win[4 * NCH + 1] = nx.y; win[4 * NCH + 2] = nx.z; win[4 * NCH + 3] = nx.w;
    uint32_t e[4 * NCH];
    byte_shift_words<4 * (NCH + 1), 4 * NCH>(win, boff, e);
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      float f;
      if (ELT == 4) f = __uint_as_float(e[i]);
      else if (std::is_same<T, __nv_bfloat16>::value) f = __uint_as_float((i & 1) ? (e[i >> 1] & 0xFFFF0000u) : (e[i >> 1] << 16));
      else f = f16_bits_to_float((i & 1) ? (e[i >> 1] >> 16) : (e[i >> 1] & 0xFFFFu));
      v[i] = (kl + i < K) ? f : 0.0f;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const ScaleInfo si = scale_from_absmax(m);
    const uint32_t ex = si.bits & 0x7C00u;
    const bool simple = (ex != 0u && ex != 0x7C00u) || si.bits == 0u;
    uint32_t words[PW];
    bool ok = simple;
#pragma unroll
    for (int p = 0; p < PW; ++p) {
      float v8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v8[i] = v[8 * p + i];
      ok = codes8<T>(v8, si.r, words[p]) && ok;
    }
    if (!__all_sync(0xffffffffu, ok)) {
      if (!ok) {
#pragma unroll
        for (int p = 0; p < PW; ++p) {
          words[p] = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) words[p] |= code_exact(v[8 * p + i], si) << (4 * i);
        }
      }
    }
    if (kl < K && (lane & (LPG - 1)) == 0) scales[crow * G + kl / (EPL * LPG)] = static_cast<uint16_t>(si.bits);
    const int64_t rowp = pshift + crow * Kp;
    const int64_t f0 = rowp + ccol * (WIN / 2);
    const int64_t hi = (f0 + WIN / 2 < rowp + Kp) ? f0 + WIN / 2 : rowp + Kp;
    store_segment<PW>(pbase, f0, f0, hi, words, lane);
  }
}

// General path, step 1: one thread per (row, group) computes the scale.
template <typename T>
__global__ void __launch_bounds__(256) quantize_scales_general_kernel(
    const T* __restrict__ w, int64_t N, int64_t K, int group, int G, uint16_t* __restrict__ scales) {
  const int64_t total = N * G;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / G;
    const int64_t g = idx - n * G;
    const int64_t k0 = g * group;
    const int64_t k1 = (k0 + group < K) ? k0 + group : K;
    float m = 0.0f;
    for (int64_t k = k0; k < k1; ++k) m = fmaxf(m, fabsf(Elem<T>::load(w + n * K + k)));
    scales[idx] = static_cast<uint16_t>(scale_from_absmax(m).bits);
  }
}

// General path, step 2: one thread per packed byte, using the stored scales.
template <typename T>
__global__ void __launch_bounds__(256) quantize_pack_general_kernel(
    const T* __restrict__ w, int64_t N, int64_t K, int group, int G,
    const uint16_t* __restrict__ scales, uint8_t* __restrict__ packed) {
  const int64_t Kp = (K + 1) >> 1;
  const int64_t total = N * Kp;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / Kp;
    const int64_t k = 2 * (idx - n * Kp);
    const ScaleInfo s0 = scale_from_bits(scales[n * G + k / group]);
    uint32_t byte = code_of(Elem<T>::load(w + n * K + k), s0);
    if (k + 1 < K) {
      const ScaleInfo s1 = scale_from_bits(scales[n * G + (k + 1) / group]);
      byte |= code_of(Elem<T>::load(w + n * K + k + 1), s1) << 4;
    }
    packed[idx] = static_cast<uint8_t>(byte);
  }
}

int grid_for(int64_t work_items, int per_block, int max_blocks_per_sm) {
  const int64_t want = (work_items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * max_blocks_per_sm;
  const int64_t g = want < cap ? want : cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <typename T>
cudaError_t launch_typed(const T* w, int64_t N, int64_t K, int group, uint8_t* packed,
                         uint16_t* scales, cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const bool aligned = (K % 8 == 0) && (reinterpret_cast<uintptr_t>(w) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(packed) % 4 == 0);
  const int lpg = group / 8;
  const bool pow2_group = (group % 8 == 0) && lpg >= 1 && lpg <= 32 && (lpg & (lpg - 1)) == 0;
  const int lpg16 = group / 16;
  const bool wide = (K % 16 == 0) && (reinterpret_cast<uintptr_t>(w) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(packed) % 8 == 0) && (group % 16 == 0) &&
                    lpg16 >= 1 && lpg16 <= 32 && (lpg16 & (lpg16 - 1)) == 0;
  if (wide) {
    const int64_t wpr = (K / 16 + 31) / 32;
    const int64_t total = N * wpr;
    const int64_t want = (total + 15) / 16;  // two windows per warp at least
    switch (lpg16) {
#define INT4_QW_CASE(L)                                                                     \
  case L:                                                                                   \
    quantize_wide_kernel<T, L><<<resident_grid(quantize_wide_kernel<T, L>, want), 256, 0,   \
                                 stream>>>(w, K, G, wpr, total, packed, scales);            \
    break;
      INT4_QW_CASE(1)
      INT4_QW_CASE(2)
      INT4_QW_CASE(4)
      INT4_QW_CASE(8)
      INT4_QW_CASE(16)
      INT4_QW_CASE(32)
#undef INT4_QW_CASE
      default:
        break;
    }
    return cudaGetLastError();
  }
  if (aligned && pow2_group) {
    const int64_t wpr = (K / 8 + 31) / 32;
    const int64_t total = N * wpr;
    const int64_t want = (total + 8 * kUnroll - 1) / (8 * kUnroll);
    switch (lpg) {
#define INT4_Q_CASE(L)                                                                       \
  case L:                                                                                    \
    quantize_aligned_kernel<T, L><<<resident_grid(quantize_aligned_kernel<T, L>, want), 256, \
                                    0, stream>>>(w, K, G, wpr, total, packed, scales);       \
    break;
      INT4_Q_CASE(1)
      INT4_Q_CASE(2)
      INT4_Q_CASE(4)
      INT4_Q_CASE(8)
      INT4_Q_CASE(16)
      INT4_Q_CASE(32)
#undef INT4_Q_CASE
      default:
        break;
    }
    return cudaGetLastError();
  }
  if (pow2_group) {
    const uintptr_t wa = reinterpret_cast<uintptr_t>(w);
    const uint8_t* wbase = reinterpret_cast<const uint8_t*>(wa & ~static_cast<uintptr_t>(15));
    const int64_t wshift = static_cast<int64_t>(wa & 15);
    const uintptr_t pa = reinterpret_cast<uintptr_t>(packed);
    uint8_t* pbase = reinterpret_cast<uint8_t*>(pa & ~static_cast<uintptr_t>(3));
    const int64_t pshift = static_cast<int64_t>(pa & 3);
    const int64_t wbytes = wshift + N * K * static_cast<int64_t>(sizeof(T));
    // kAnyChunks16 16-byte chunks per lane for 16-bit weights when a group
    // spans whole lanes.
    constexpr int kWideEpl = 8 * kAnyChunks16;
    const bool two = sizeof(T) == 2 && group % kWideEpl == 0 && group / kWideEpl <= 32;
    const int epl = two ? kWideEpl : 8;
    const int lanes = group / epl;
    const int64_t wpr = (K + 32 * epl - 1) / (32 * epl);
    const int64_t total = N * wpr;
    const int64_t want = (total + 31) / 32;
#define INT4_QA_CASE(L, C)                                                                     \
  case L:                                                                                      \
    quantize_any_kernel<T, L, C><<<resident_grid(quantize_any_kernel<T, L, C>, want), 256, 0,  \
                                   stream>>>(reinterpret_cast<const uint8_t*>(wbase), wshift,  \
                                             wbytes, K, G, wpr, total, pbase, pshift, scales); \
    break;
    if (two) {
      switch (lanes) {
        INT4_QA_CASE(1, kAnyChunks16)
        INT4_QA_CASE(2, kAnyChunks16)
        INT4_QA_CASE(4, kAnyChunks16)
        INT4_QA_CASE(8, kAnyChunks16)
        INT4_QA_CASE(16, kAnyChunks16)
        INT4_QA_CASE(32, kAnyChunks16)
        default:
          break;
      }
    } else {
      constexpr int kC = sizeof(T) == 4 ? 2 : 1;  // 8 elements per lane
      switch (lanes) {
        INT4_QA_CASE(1, kC)
        INT4_QA_CASE(2, kC)
        INT4_QA_CASE(4, kC)
        INT4_QA_CASE(8, kC)
        INT4_QA_CASE(16, kC)
        INT4_QA_CASE(32, kC)
        default:
          break;
      }
    }
#undef INT4_QA_CASE
    return cudaGetLastError();
  }
  quantize_scales_general_kernel<T><<<grid_for(N * G, 256, 16), 256, 0, stream>>>(w, N, K, group, G,
                                                                                    scales);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t Kp = (K + 1) / 2;
  quantize_pack_general_kernel<T><<<grid_for(N * Kp, 256, 16), 256, 0, stream>>>(w, N, K, group, G,
                                                                                   scales, packed);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* w, DType wt, int64_t N, int64_t K, int group,
                            uint8_t* packed, uint16_t* scales, cudaStream_t stream) {
  switch (wt) {
    case DType::F32:
      return launch_typed(static_cast<const float*>(w), N, K, group, packed, scales, stream);
    case DType::BF16:
      return launch_typed(static_cast<const __nv_bfloat16*>(w), N, K, group, packed, scales,
                          stream);
    case DType::F16:
      return launch_typed(static_cast<const __half*>(w), N, K, group, packed, scales, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace int4lib
