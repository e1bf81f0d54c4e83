// General dequantizing matmul on CUDA cores (sm_100a): any K, any group,
// any alignment, fp32 / bf16 / fp16 activations.
//
// y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * q[n, k]), the order of
// the int4_matmul function of the page "Implement INT4 group quantization,
// nibble packing and a dequantizing matmul" (problem statement): integer
// weights times x first, then the group's scale per output column.
//
// Each thread keeps an fp32 partial sum over a run of at most 32 consecutive
// k inside one group (each step x * q + partial is one correctly rounded
// FMA; q is an exact small integer), and folds every run into an fp64 running
// sum after multiplying it by the group's scale.  The worst-case error is then
// below 32 fp32 roundings of sum |x||w_hat| (< 2e-6 relative), inside the
// 1e-5 bound for fp32 activations for any K and group.
//
// This is the correctness kernel for shapes and dtypes the tensor-core kernels
// do not take; it tiles 64 weight rows x 16 activation rows per block with a
// 32-wide K step staged through shared memory.  For the asymmetric scheme of
// the page "Build a Blockwise INT4 Inference Engine" (step 2) the staged codes
// are unsigned and the group's zero point is subtracted at use (q - z is an
// exact small integer too); the optional bias and ReLU apply at the store.
#include "common.cuh"
#include "internal.h"

namespace int4lib {

namespace {

constexpr int BN = 64;   // weight rows per block
constexpr int BM = 16;   // activation rows per block
constexpr int BK = 32;   // k per shared-memory step
constexpr int TM = 4;    // activation rows per thread (BM / (256 / BN))

template <typename TX, bool ASYM>
__global__ void __launch_bounds__(256) matmul_simt_kernel(
    const TX* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t K, int group,
    int G, int64_t M, int64_t N, Epilogue ep, float* __restrict__ y) {
  __shared__ float xs[BM][BK + 1];
  __shared__ int8_t qs[BN][BK + 4];

  const int tid = threadIdx.x;
  const int tn = tid % BN;
  const int tm = tid / BN;  // 0..3
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t Kp = (K + 1) >> 1;
  const int64_t n = n0 + tn;

  double acc[TM];
  float part[TM];
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    acc[i] = 0.0;
    part[i] = 0.0f;
  }
  float cur_scale = 0.0f;
  float cur_zero = 0.0f;

  for (int64_t k0 = 0; k0 < K; k0 += BK) {
    // Stage x[m0 : m0+16, k0 : k0+32] as fp32 (zeros outside the matrix).
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int64_t m = m0 + r, k = k0 + c;
      xs[r][c] = (m < M && k < K) ? Elem<TX>::load(x + m * K + k) : 0.0f;
    }
    // Stage q[n0 : n0+64, k0 : k0+32] sign-extended (zeros outside).
    {
      const int r = tid / 4;
      const int c0 = (tid % 4) * 8;
      const int64_t nr = n0 + r;
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const int64_t k = k0 + c0 + j;  // even
        uint32_t byte = 0;
        if (nr < N && k < K) byte = __ldg(packed + nr * Kp + (k >> 1));
        if (ASYM) {
          qs[r][c0 + j] = static_cast<int8_t>(byte & 0xFu);
          qs[r][c0 + j + 1] = (k + 1 < K) ? static_cast<int8_t>(byte >> 4) : 0;
        } else {
          qs[r][c0 + j] = static_cast<int8_t>(static_cast<int32_t>(byte << 28) >> 28);
          qs[r][c0 + j + 1] =
              (k + 1 < K) ? static_cast<int8_t>(static_cast<int32_t>(byte << 24) >> 28) : 0;
        }
      }
    }
    __syncthreads();

    const int kend = (K - k0 < BK) ? static_cast<int>(K - k0) : BK;
    for (int c = 0; c < kend; ++c) {
      const int64_t k = k0 + c;
      if (c == 0 || k % group == 0) {
        // A new run starts: fold the previous run with its group's scale.
#pragma unroll
        for (int i = 0; i < TM; ++i) {
          acc[i] += static_cast<double>(part[i]) * static_cast<double>(cur_scale);
          part[i] = 0.0f;
        }
        cur_scale = (n < N) ? f16_bits_to_float(__ldg(scales + n * G + k / group)) : 0.0f;
        if (ASYM) cur_zero = (n < N) ? static_cast<float>(__ldg(zeros + n * G + k / group)) : 0.0f;
      }
      const float q = static_cast<float>(qs[tn][c]) - cur_zero;  // exact
#pragma unroll
      for (int i = 0; i < TM; ++i) part[i] = fmaf(xs[tm * TM + i][c], q, part[i]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    acc[i] += static_cast<double>(part[i]) * static_cast<double>(cur_scale);
    const int64_t m = m0 + tm * TM + i;
    if (m < M && n < N) y[m * N + n] = ep.apply(static_cast<float>(acc[i]), n);
  }
}

template <typename TX>
void launch_tx(const TX* x, const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
               int64_t K, int group, int G, int64_t M, int64_t N, const Epilogue& ep, float* y,
               dim3 grid, cudaStream_t stream) {
  if (zeros != nullptr)
    matmul_simt_kernel<TX, true><<<grid, 256, 0, stream>>>(x, packed, scales, zeros, K, group, G, M,
                                                           N, ep, y);
  else
    matmul_simt_kernel<TX, false><<<grid, 256, 0, stream>>>(x, packed, scales, nullptr, K, group, G,
                                                            M, N, ep, y);
}

}  // namespace

cudaError_t launch_matmul_simt(const void* x, DType xt, const uint8_t* packed,
                               const uint16_t* scales, const uint8_t* zeros, int64_t K, int group,
                               int64_t M, int64_t N, const Epilogue& ep, float* y,
                               cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const int64_t gx = (N + BN - 1) / BN;
  const int64_t gy = (M + BM - 1) / BM;
  if (gx > 0x7fffffff || gy > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  switch (xt) {
    case DType::F32:
      launch_tx(static_cast<const float*>(x), packed, scales, zeros, K, group, G, M, N, ep, y, grid,
                stream);
      break;
    case DType::BF16:
      launch_tx(static_cast<const __nv_bfloat16*>(x), packed, scales, zeros, K, group, G, M, N, ep,
                y, grid, stream);
      break;
    case DType::F16:
      launch_tx(static_cast<const __half*>(x), packed, scales, zeros, K, group, G, M, N, ep, y,
                grid, stream);
      break;
  }
  return cudaGetLastError();
}

}  // namespace int4lib
