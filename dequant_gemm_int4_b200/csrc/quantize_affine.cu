// Asymmetric (affine) 4-bit quantization with per-group zero points (sm_100a).
//
// Follows step 2 of the page "Build a Blockwise INT4 Inference Engine": per
// row and K-group, scale = (max - min) / 15, zero point = clip(round(-min /
// scale), 0, 15), q = clip(round(w / scale + zero point), 0, 15).  Layout as
// the symmetric scheme's: the unsigned code of element 2j in the low nibble
// of byte j (zero pad nibble for odd K), fp16 scales [N, G], and uint8 zero
// points [N, G].  Rounding convention, in the page's order of operations:
// d = fp32(max - min), s = fp16_RNE(fp32(d / 15)); with sf = fp32(s),
// z = clip(rint(fp32(-min / sf)), 0, 15) and q = clip(rint(fp32(fp32(w / sf)
// + z)), 0, 15), every division an IEEE fp32 division and rint half to even.
// A zero scale (a constant group, or a range that underflows fp16) codes the
// group as q = 0, z = 0.
//
// A warp takes a window of 512
// consecutive weights of one row (16 per lane, two 16- or 32-byte loads),
// reduces the group's min and max with shuffles over its group / 16 lanes,
// codes the weights two per instruction (float2 arithmetic) and stores 8
// packed bytes per lane.  It reads w once but runs at about half of HBM
// bandwidth: the ALU pipe (the clamp and the min/max of every weight) bounds
// it.  Groups of 8 take windows of 256 (8 per lane); any other shape takes a
// two-kernel general path (scales and zero points, then one thread per
// packed byte).
#include "common.cuh"
#include "internal.h"

namespace int4lib {

namespace {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}
template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = f16_bits_to_float(w[i] & 0xFFFFu);
    v[2 * i + 1] = f16_bits_to_float(w[i] >> 16);
  }
}

struct Affine {
  float sf;       // the scale, read back from fp16
  float r;        // 1 / sf correctly rounded (0 when sf is 0)
  float zf;       // the zero point as a float (an integer 0..15)
  uint32_t bits;  // the fp16 scale
  uint32_t z;
};

// fp32(v / sf), correctly rounded, from r = RN(1 / sf): q = RN(v r) is within
// one ulp of the quotient, the residual v - q sf is exact by FMA, and
// RN(q + residual r) is the correctly rounded quotient (Markstein's theorem
// for a correctly rounded reciprocal; the test suite compares the codes with
// the IEEE division bit for bit).  Quotients of 2^100 or more, and an
// infinite scale, take the IEEE division, where the residual could overflow.  The residual is exact
// whenever the quotient is 1/4 or more (then |v| >= 2^-26, sf being at least
// 2^-24); a smaller quotient cannot move rint(quotient + z), exact or not.
__device__ __forceinline__ float div_by_scale(float v, float sf, float r) {
  const float q = __fmul_rn(v, r);
  if (!(fabsf(q) < 0x1p100f) || r == 0.0f) return __fdiv_rn(v, sf);  // huge, or sf = +inf
  const float e = __fmaf_rn(-q, sf, v);
  return __fmaf_rn(e, r, q);
}

// fp32(d / 15), correctly rounded, for finite d >= 0: Markstein's step with
// the constant c = RN(1/15) (q0 = d c, exact residual d - 15 q0 by FMA,
// q0 + residual c).  Where the residual could round (d subnormal), the
// quotient lies far below the smallest fp16 subnormal and the scale is 0
// either way.  The test suite compares the scales with the IEEE division on
// every fp32 mantissa of the binades that matter.
__device__ __forceinline__ float div15_rn(float d) {
  const float c = 0.0666666701f;  // fp32 nearest to 1/15
  const float q0 = __fmul_rn(d, c);
  const float e = __fmaf_rn(-15.0f, q0, d);
  return __fmaf_rn(e, c, q0);
}

// Scale and zero point of a group with extremes mn <= mx.
__device__ __forceinline__ Affine affine_params(float mn, float mx) {
  Affine a;
  const float d = __fsub_rn(mx, mn);
  a.bits = __half_as_ushort(__float2half_rn(div15_rn(d)));
  a.sf = f16_bits_to_float(a.bits);
  a.r = a.sf != 0.0f ? __frcp_rn(a.sf) : 0.0f;
  a.zf = 0.0f;
  if (a.sf != 0.0f) {
    const float t = rintf(div_by_scale(-mn, a.sf, a.r));
    a.zf = fminf(fmaxf(t, 0.0f), 15.0f);
  }
  a.z = static_cast<uint32_t>(a.zf);
  return a;
}

__device__ __forceinline__ Affine affine_from_stored(uint16_t bits, uint8_t z) {
  Affine a;
  a.bits = bits;
  a.sf = f16_bits_to_float(bits);
  a.r = a.sf != 0.0f ? __frcp_rn(a.sf) : 0.0f;
  a.z = z;
  a.zf = static_cast<float>(z);
  return a;
}

// The unsigned code of v: clip(rint(fp32(fp32(v / sf) + z)), 0, 15); 0 when
// the scale is 0.
__device__ __forceinline__ uint32_t affine_code(float v, const Affine& a) {
  if (a.sf == 0.0f) return 0u;
  const float u = __fadd_rn(div_by_scale(v, a.sf, a.r), a.zf);
  return static_cast<uint32_t>(fminf(fmaxf(rintf(u), 0.0f), 15.0f));
}

// The same code for a group whose every |v| * r stays below 2^99 (checked
// once per group), with a finite non-zero scale: the quotient by Markstein's
// step with no overflow test, the clamp before the rounding (the same
// result: the bounds are integers), and rint as the exact addition of
// 1.5 * 2^23, whose low mantissa bits then hold the code.
__device__ __forceinline__ uint32_t affine_code_fast(float v, const Affine& a) {
  const float q = __fmul_rn(v, a.r);
  const float e = __fmaf_rn(-q, a.sf, v);
  const float u = __fadd_rn(__fmaf_rn(e, a.r, q), a.zf);
  const float uc = fminf(fmaxf(u, 0.0f), 15.0f);
  return __float_as_uint(__fadd_rn(uc, 12582912.0f)) & 0xFu;
}

// affine_code_fast on 16 weights, two per float2 instruction (each component
// rounds as the scalar operation does): element 2j in the low nibble of
// byte j, bytes 0..3 in .x and 4..7 in .y.
__device__ __forceinline__ uint2 affine_codes16_fast(const float (&v)[16], const Affine& a) {
  const float2 r2 = make_float2(a.r, a.r);
  const float2 ns2 = make_float2(-a.sf, -a.sf);
  const float2 z2 = make_float2(a.zf, a.zf);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  uint32_t word[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 x = make_float2(v[2 * i], v[2 * i + 1]);
    const float2 q = __fmul2_rn(x, r2);
    const float2 e = __ffma2_rn(q, ns2, x);  // x - q sf, exact
    const float2 u = __fadd2_rn(__ffma2_rn(e, r2, q), z2);
    const float2 uc = make_float2(fminf(fmaxf(u.x, 0.0f), 15.0f), fminf(fmaxf(u.y, 0.0f), 15.0f));
    const float2 t = __fadd2_rn(uc, magic);
    const uint32_t byte = (__float_as_uint(t.x) & 0xFu) | ((__float_as_uint(t.y) & 0xFu) << 4);
    word[i >> 2] |= byte << (8 * (i & 3));
  }
  return make_uint2(word[0], word[1]);
}

// Fast path: K % 8 == 0, group = 8 LPG with LPG a power of two <= 32, w
// 16-byte aligned, packed 4-byte aligned.  Windows (256 weights of one row)
// are numbered row-major; each warp takes a contiguous range of them.
template <typename T, int LPG>
__global__ void __launch_bounds__(256) quantize_affine_window_kernel(
    const T* __restrict__ w, int64_t K, int G, int64_t windows_per_row, int64_t total_windows,
    uint8_t* __restrict__ packed, uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t per = (total_windows + nwarps - 1) / nwarps;
  const int64_t wbeg = warp * per;
  const int64_t wend = (wbeg + per < total_windows) ? wbeg + per : total_windows;
  if (wbeg >= wend) return;
  int64_t row = wbeg / windows_per_row;
  int64_t win = wbeg - row * windows_per_row;
  // The next window's weights are loaded while this one is coded, so that
  // every warp keeps two loads in flight.
  auto load_window = [&](int64_t r, int64_t wn, float (&dst)[8]) {
    const int64_t k = wn * 256 + 8 * lane;
    if (k < K) {
      load8<T>(w + r * K + k, dst);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = 0.0f;
    }
  };
  float vnext[8];
  load_window(row, win, vnext);
  for (int64_t wi = wbeg; wi < wend; ++wi) {
    const int64_t k0 = win * 256 + 8 * lane;
    const bool active = k0 < K;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = vnext[i];
    if (wi + 1 < wend) {
      const bool wrap = win + 1 == windows_per_row;
      load_window(wrap ? row + 1 : row, wrap ? 0 : win + 1, vnext);
    }
    float mn = active ? v[0] : __int_as_float(0x7F800000);   // +inf
    float mx = active ? v[0] : __int_as_float(0xFF800000);   // -inf
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      mn = fminf(mn, active ? v[i] : mn);
      mx = fmaxf(mx, active ? v[i] : mx);
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (active) {
      const Affine a = affine_params(mn, mx);
      uint32_t word = 0u;
      const bool fast = a.sf != 0.0f && a.r != 0.0f &&
                        __fmul_rn(fmaxf(fabsf(mn), fabsf(mx)), a.r) < 0x1p99f;
      if (fast) {
#pragma unroll
        for (int i = 0; i < 8; ++i) word |= affine_code_fast(v[i], a) << (4 * i);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) word |= affine_code(v[i], a) << (4 * i);
      }
      *reinterpret_cast<uint32_t*>(packed + row * (K >> 1) + (k0 >> 1)) = word;
      if ((lane & (LPG - 1)) == 0) {
        const int64_t gi = row * G + k0 / (8 * LPG);
        scales[gi] = static_cast<uint16_t>(a.bits);
        zeros[gi] = static_cast<uint8_t>(a.z);
      }
    }
    if (++win == windows_per_row) {
      win = 0;
      ++row;
    }
  }
}

// Wide fast path: K % 16 == 0, group = 16 LPG with LPG a power of two <= 32,
// w 16-byte aligned, packed 8-byte aligned.  Windows (512 weights of one
// row, 16 per lane) are numbered row-major; each warp takes a contiguous
// range of them.  Lanes past the row's end (K not a multiple of 512) take
// part in the shuffles with neutral extremes and store nothing.
template <typename T, int LPG>
__global__ void __launch_bounds__(256) quantize_affine_wide_kernel(
    const T* __restrict__ w, int64_t K, int G, int64_t windows_per_row, int64_t total_windows,
    uint8_t* __restrict__ packed, uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros) {
  constexpr int kGroup = 16 * LPG;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t per = (total_windows + nwarps - 1) / nwarps;
  const int64_t wbeg = warp * per;
  const int64_t wend = (wbeg + per < total_windows) ? wbeg + per : total_windows;
  if (wbeg >= wend) return;
  int64_t row = wbeg / windows_per_row;
  int64_t win = wbeg - row * windows_per_row;
  // The next window's weights are loaded while this one is coded.
  auto load_window = [&](int64_t r, int64_t wn, float (&dst)[16]) {
    const int64_t k = wn * 512 + 16 * lane;
    if (k < K) {
      float lo[8], hi[8];
      load8<T>(w + r * K + k, lo);
      load8<T>(w + r * K + k + 8, hi);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dst[i] = lo[i];
        dst[8 + i] = hi[i];
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[i] = 0.0f;
    }
  };
  float vnext[16];
  load_window(row, win, vnext);
  for (int64_t wi = wbeg; wi < wend; ++wi) {
    const int64_t k0 = win * 512 + 16 * lane;
    const bool active = k0 < K;
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = vnext[i];
    if (wi + 1 < wend) {
      const bool wrap = win + 1 == windows_per_row;
      load_window(wrap ? row + 1 : row, wrap ? 0 : win + 1, vnext);
    }
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      mn = fminf(mn, v[i]);
      mx = fmaxf(mx, v[i]);
    }
    if (!active) {
      mn = __int_as_float(0x7F800000);  // +inf
      mx = __int_as_float(0xFF800000);  // -inf
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (active) {
      const Affine a = affine_params(mn, mx);
      const bool fast = a.sf != 0.0f && a.r != 0.0f &&
                        __fmul_rn(fmaxf(fabsf(mn), fabsf(mx)), a.r) < 0x1p99f;
      uint2 word;
      if (fast) {
        word = affine_codes16_fast(v, a);
      } else {
        word = make_uint2(0u, 0u);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          word.x |= affine_code(v[i], a) << (4 * i);
          word.y |= affine_code(v[8 + i], a) << (4 * i);
        }
      }
      *reinterpret_cast<uint2*>(packed + row * (K >> 1) + (k0 >> 1)) = word;
      if ((lane & (LPG - 1)) == 0) {
        const int64_t gi = row * G + k0 / kGroup;
        scales[gi] = static_cast<uint16_t>(a.bits);
        zeros[gi] = static_cast<uint8_t>(a.z);
      }
    }
    if (++win == windows_per_row) {
      win = 0;
      ++row;
    }
  }
}

// General path, step 1: one thread per (row, group).
template <typename T>
__global__ void __launch_bounds__(256) quantize_affine_params_kernel(
    const T* __restrict__ w, int64_t N, int64_t K, int group, int G, uint16_t* __restrict__ scales,
    uint8_t* __restrict__ zeros) {
  const int64_t total = N * G;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / G;
    const int64_t k0 = (idx - n * G) * group;
    const int64_t k1 = (k0 + group < K) ? k0 + group : K;
    float mn = Elem<T>::load(w + n * K + k0), mx = mn;
    for (int64_t k = k0 + 1; k < k1; ++k) {
      const float v = Elem<T>::load(w + n * K + k);
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
    const Affine a = affine_params(mn, mx);
    scales[idx] = static_cast<uint16_t>(a.bits);
    zeros[idx] = static_cast<uint8_t>(a.z);
  }
}

// General path, step 2: one thread per packed byte, from the stored scale
// and zero point.
template <typename T>
__global__ void __launch_bounds__(256) quantize_affine_pack_kernel(
    const T* __restrict__ w, int64_t N, int64_t K, int group, int G,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros,
    uint8_t* __restrict__ packed) {
  const int64_t Kp = (K + 1) >> 1;
  const int64_t total = N * Kp;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / Kp;
    const int64_t k = 2 * (idx - n * Kp);
    const int64_t g0 = n * G + k / group;
    uint32_t byte = affine_code(Elem<T>::load(w + n * K + k), affine_from_stored(scales[g0], zeros[g0]));
    if (k + 1 < K) {
      const int64_t g1 = n * G + (k + 1) / group;
      byte |= affine_code(Elem<T>::load(w + n * K + k + 1), affine_from_stored(scales[g1], zeros[g1]))
              << 4;
    }
    packed[idx] = static_cast<uint8_t>(byte);
  }
}

template <typename T, int LPG>
cudaError_t launch_window(const T* w, int64_t N, int64_t K, int G, uint8_t* packed,
                          uint16_t* scales, uint8_t* zeros, cudaStream_t stream) {
  const int64_t wpr = (K + 255) / 256;
  const int64_t total = N * wpr;
  const int grid = resident_grid(quantize_affine_window_kernel<T, LPG>, (total + 7) / 8);
  quantize_affine_window_kernel<T, LPG><<<grid, 256, 0, stream>>>(w, K, G, wpr, total, packed,
                                                                  scales, zeros);
  return cudaGetLastError();
}

template <typename T, int LPG>
cudaError_t launch_wide(const T* w, int64_t N, int64_t K, int G, uint8_t* packed,
                        uint16_t* scales, uint8_t* zeros, cudaStream_t stream) {
  const int64_t wpr = (K + 511) / 512;
  const int64_t total = N * wpr;
  const int grid = resident_grid(quantize_affine_wide_kernel<T, LPG>, (total + 7) / 8);
  quantize_affine_wide_kernel<T, LPG><<<grid, 256, 0, stream>>>(w, K, G, wpr, total, packed,
                                                                scales, zeros);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const T* w, int64_t N, int64_t K, int group, uint8_t* packed,
                         uint16_t* scales, uint8_t* zeros, cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const bool wide = K % 16 == 0 && reinterpret_cast<uintptr_t>(w) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(packed) % 8 == 0;
  if (wide) {
    switch (group) {
      case 16: return launch_wide<T, 1>(w, N, K, G, packed, scales, zeros, stream);
      case 32: return launch_wide<T, 2>(w, N, K, G, packed, scales, zeros, stream);
      case 64: return launch_wide<T, 4>(w, N, K, G, packed, scales, zeros, stream);
      case 128: return launch_wide<T, 8>(w, N, K, G, packed, scales, zeros, stream);
      case 256: return launch_wide<T, 16>(w, N, K, G, packed, scales, zeros, stream);
      case 512: return launch_wide<T, 32>(w, N, K, G, packed, scales, zeros, stream);
      default: break;
    }
  }
  const bool fast = K % 8 == 0 && reinterpret_cast<uintptr_t>(w) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(packed) % 4 == 0;
  if (fast) {
    switch (group) {
      case 8: return launch_window<T, 1>(w, N, K, G, packed, scales, zeros, stream);
      case 16: return launch_window<T, 2>(w, N, K, G, packed, scales, zeros, stream);
      case 32: return launch_window<T, 4>(w, N, K, G, packed, scales, zeros, stream);
      case 64: return launch_window<T, 8>(w, N, K, G, packed, scales, zeros, stream);
      case 128: return launch_window<T, 16>(w, N, K, G, packed, scales, zeros, stream);
      case 256: return launch_window<T, 32>(w, N, K, G, packed, scales, zeros, stream);
      default: break;
    }
  }
  quantize_affine_params_kernel<T><<<resident_grid(quantize_affine_params_kernel<T>, (N * G + 255) / 256),
                                     256, 0, stream>>>(w, N, K, group, G, scales, zeros);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t Kp = (K + 1) / 2;
  quantize_affine_pack_kernel<T><<<resident_grid(quantize_affine_pack_kernel<T>, (N * Kp + 255) / 256),
                                   256, 0, stream>>>(w, N, K, group, G, scales, zeros, packed);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_affine(const void* w, DType wt, int64_t N, int64_t K, int group,
                                   uint8_t* packed, uint16_t* scales, uint8_t* zeros,
                                   cudaStream_t stream) {
  switch (wt) {
    case DType::F32:
      return launch_typed(static_cast<const float*>(w), N, K, group, packed, scales, zeros, stream);
    case DType::BF16:
      return launch_typed(static_cast<const __nv_bfloat16*>(w), N, K, group, packed, scales, zeros,
                          stream);
    case DType::F16:
      return launch_typed(static_cast<const __half*>(w), N, K, group, packed, scales, zeros, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace int4lib
