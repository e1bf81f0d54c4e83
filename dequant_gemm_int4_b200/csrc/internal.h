// Internal launcher interface between the C-ABI layer (int4_abi.cu) and the
// kernels.  Each launcher assumes its arguments were validated by the ABI
// layer and returns a cudaError_t from the launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace int4lib {

enum class DType : int { F32 = 0, BF16 = 1, F16 = 2 };

inline int dtype_size(DType t) { return t == DType::F32 ? 4 : 2; }

// Device-side status word: kernels whose bounded waits give up set a bit.
constexpr uint32_t kStatusTimeout = 1u;
cudaError_t read_and_clear_status(uint32_t* out, cudaStream_t stream);
// Device address of the status word on the current device (nullptr on error).
uint32_t* status_word();
cudaError_t launch_wait_timeout_selftest(uint32_t spins, cudaStream_t stream);

// quantize.cu
cudaError_t launch_quantize(const void* w, DType wt, int64_t N, int64_t K, int group,
                            uint8_t* packed, uint16_t* scales, cudaStream_t stream);
// quantize_affine.cu: the asymmetric variant (unsigned codes, zero points).
cudaError_t launch_quantize_affine(const void* w, DType wt, int64_t N, int64_t K, int group,
                                   uint8_t* packed, uint16_t* scales, uint8_t* zeros,
                                   cudaStream_t stream);
// unpack.cu
cudaError_t launch_unpack(const uint8_t* packed, int64_t K, int64_t N, int8_t* out,
                          cudaStream_t stream);
// dequantize.cu: w_hat = q * s (zeros == nullptr) or (q - z) * s, rounded to
// the output type.
cudaError_t launch_dequantize(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                              int64_t K, int group, int64_t N, void* out, DType ot,
                              cudaStream_t stream);
// matmul_simt.cu
cudaError_t launch_matmul_simt(const void* x, DType xt, const uint8_t* packed,
                               const uint16_t* scales, const uint8_t* zeros, int64_t K, int group,
                               int64_t M, int64_t N, const Epilogue& ep, float* y,
                               cudaStream_t stream);
// matmul_decode.cu
bool decode_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                      const uint8_t* packed);
// Bytes of caller workspace the decode path needs for this problem on the
// current device (0: none); the schedule int4_matmul_ws runs with it.
cudaError_t decode_workspace_size(DType xt, int64_t K, int group, int64_t M, int64_t N,
                                  size_t* bytes);
// The decode matmul.  workspace == nullptr with workspace_bytes == 0: the
// schedule that needs no scratch.  Otherwise the workspace (zero-filled
// before its first use, 256-byte aligned) must hold decode_workspace_size
// bytes, else cudaErrorInvalidValue with *need set.
cudaError_t launch_matmul_decode(const void* x, DType xt, const uint8_t* packed,
                                 const uint16_t* scales, const uint8_t* zeros, const Epilogue& ep,
                                 int64_t K, int group, int64_t M, int64_t N, float* y,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream,
                                 size_t* need);
// The same decode matmul with its scratch in the library's fixed device
// array (no allocation).  cudaErrorInvalidValue with *need set: the array is
// too small for this call.
cudaError_t launch_matmul_decode_noalloc(const void* x, DType xt, const uint8_t* packed,
                                         const uint16_t* scales, int64_t K, int group, int64_t M,
                                         int64_t N, float* y, cudaStream_t stream, size_t* need);
size_t decode_noalloc_scratch_bytes();
// Zeroes the arrival counters of the fixed array on the current device
// (after a device-side wait gave up); synchronizes the device.
cudaError_t reset_split_counters();
// matmul_prefill.cu
bool prefill_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                       const uint8_t* packed);
// With a workspace of prefill_workspace_size bytes (when that is non-zero:
// fewer tiles than SMs), K is split into pieces whose fp32 sums a second
// kernel adds; a smaller or null workspace runs the call unsplit.  The sums
// start kWorkspaceCounterBytes into the workspace: a workspace also serves
// decode calls, whose layout begins with arrival counters that every call
// must find zero (1024 counters of 4 bytes in matmul_decode.cu).
cudaError_t launch_matmul_prefill(const void* x, DType xt, const uint8_t* packed,
                                  const uint16_t* scales, const uint8_t* zeros, const Epilogue& ep,
                                  int64_t K, int group, int64_t M, int64_t N, float* y,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream);
size_t prefill_workspace_size(int64_t K, int group, int64_t M, int64_t N);
constexpr size_t kWorkspaceCounterBytes = 4096;

int num_sms();  // SM count of the current device (cached per device)

// Grid of at most one resident wave of `kern` (256-thread blocks, no dynamic
// shared memory) for kernels whose blocks take equal contiguous shares of the
// work, so no partial last wave trails the others.
template <typename Kern>
int resident_grid(Kern kern, int64_t want) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int64_t g = want < cap ? want : cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace int4lib
