// C-ABI entry points of the INT4 library: argument validation, kernel choice,
// error reporting.  Declarations and the contract are in include/int4.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <mutex>
#include <string>

#include "int4.h"
#include "common.cuh"
#include "internal.h"

namespace int4lib {

namespace {

// One status word per device that loads the library.
__device__ uint32_t g_int4_status = 0;

thread_local std::string t_last_error;

int fail(int code, const char* msg) {
  t_last_error = msg;
  return code;
}

int fail_cuda(cudaError_t e, const char* where) {
  t_last_error = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return INT4_ERR_CUDA;
}

bool dtype_ok(int32_t t) { return t == INT4_DTYPE_F32 || t == INT4_DTYPE_BF16 || t == INT4_DTYPE_F16; }

bool mul_ok(int64_t a, int64_t b) {
  // a, b >= 0; product below 2^62.
  if (a == 0 || b == 0) return true;
  return a <= (static_cast<int64_t>(1) << 62) / b;
}

bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

// Spins on an mbarrier that nothing completes, with an iteration limit; on
// giving up it records a timeout in the status word and returns.
__global__ void wait_timeout_selftest_kernel(uint32_t spins, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(1));
    asm volatile("fence.mbarrier_init.release.cluster;");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t done = 0;
    for (uint32_t i = 0; i < spins && !done; ++i) {
      asm volatile(
          "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
          " selp.u32 %0, 1, 0, p;\n}"
          : "=r"(done)
          : "r"(addr), "r"(0u));
    }
    if (!done) report_status(status, kStatusTimeout);
  }
}

}  // namespace

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

uint32_t* status_word() {
  static std::mutex mu;
  static uint32_t* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_int4_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<uint32_t*>(p);
  }
  return cache[dev];
}

cudaError_t read_and_clear_status(uint32_t* out, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(out, g_int4_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_int4_status, &zero, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  if (*out & kStatusTimeout) return reset_split_counters();
  return cudaSuccess;
}

cudaError_t launch_wait_timeout_selftest(uint32_t spins, cudaStream_t stream) {
  uint32_t* st = status_word();
  if (st == nullptr) return cudaErrorInvalidSymbol;
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(spins, st);
  return cudaGetLastError();
}

}  // namespace int4lib

using int4lib::DType;

extern "C" {

int int4_version(void) { return 1 * 10000 + 0 * 100 + 0; }

const char* int4_last_error(void) { return int4lib::t_last_error.c_str(); }

int int4_quantize(const void* w, int32_t w_dtype, int64_t N, int64_t K, int32_t group,
                  uint8_t* packed, uint16_t* scales, void* stream) {
  if (!int4lib::dtype_ok(w_dtype)) return int4lib::fail(INT4_ERR_DTYPE, "int4_quantize: unknown w_dtype");
  if (N < 0 || K < 1 || group < 1)
    return int4lib::fail(INT4_ERR_ARG, "int4_quantize: need N >= 0, K >= 1, group >= 1");
  if (!int4lib::mul_ok(N, K)) return int4lib::fail(INT4_ERR_ARG, "int4_quantize: N*K too large");
  if (N == 0) return INT4_OK;
  if (!w || !packed || !scales) return int4lib::fail(INT4_ERR_ARG, "int4_quantize: null pointer");
  const DType t = static_cast<DType>(w_dtype);
  if (!int4lib::aligned(w, int4lib::dtype_size(t)) || !int4lib::aligned(scales, 2))
    return int4lib::fail(INT4_ERR_ALIGN, "int4_quantize: w or scales not aligned to its element size");
  const cudaError_t e = int4lib::launch_quantize(w, t, N, K, group, packed, scales,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_quantize");
}

int int4_unpack(const uint8_t* packed, int64_t K, int64_t N, int8_t* out, void* stream) {
  if (N < 0 || K < 1) return int4lib::fail(INT4_ERR_ARG, "int4_unpack: need N >= 0, K >= 1");
  if (!int4lib::mul_ok(N, K)) return int4lib::fail(INT4_ERR_ARG, "int4_unpack: N*K too large");
  if (N == 0) return INT4_OK;
  if (!packed || !out) return int4lib::fail(INT4_ERR_ARG, "int4_unpack: null pointer");
  const cudaError_t e = int4lib::launch_unpack(packed, K, N, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_unpack");
}

int int4_quantize_affine(const void* w, int32_t w_dtype, int64_t N, int64_t K, int32_t group,
                         uint8_t* packed, uint16_t* scales, uint8_t* zeros, void* stream) {
  if (!int4lib::dtype_ok(w_dtype)) return int4lib::fail(INT4_ERR_DTYPE, "int4_quantize_affine: unknown w_dtype");
  if (N < 0 || K < 1 || group < 1)
    return int4lib::fail(INT4_ERR_ARG, "int4_quantize_affine: need N >= 0, K >= 1, group >= 1");
  if (!int4lib::mul_ok(N, K)) return int4lib::fail(INT4_ERR_ARG, "int4_quantize_affine: N*K too large");
  if (N == 0) return INT4_OK;
  if (!w || !packed || !scales || !zeros)
    return int4lib::fail(INT4_ERR_ARG, "int4_quantize_affine: null pointer");
  const DType t = static_cast<DType>(w_dtype);
  if (!int4lib::aligned(w, int4lib::dtype_size(t)) || !int4lib::aligned(scales, 2))
    return int4lib::fail(INT4_ERR_ALIGN, "int4_quantize_affine: w or scales not aligned to its element size");
  const cudaError_t e = int4lib::launch_quantize_affine(w, t, N, K, group, packed, scales, zeros,
                                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_quantize_affine");
}

static int dequantize_common(const char* name, const uint8_t* packed, const uint16_t* scales,
                             const uint8_t* zeros, bool need_zeros, int64_t K, int32_t group,
                             int64_t N, void* out, int32_t out_dtype, void* stream) {
  char msg[160];
  if (!int4lib::dtype_ok(out_dtype)) {
    std::snprintf(msg, sizeof msg, "%s: unknown out_dtype", name);
    return int4lib::fail(INT4_ERR_DTYPE, msg);
  }
  if (N < 0 || K < 1 || group < 1 || !int4lib::mul_ok(N, K)) {
    std::snprintf(msg, sizeof msg, "%s: need N >= 0, K >= 1, group >= 1 and N*K below 2^62", name);
    return int4lib::fail(INT4_ERR_ARG, msg);
  }
  if (N == 0) return INT4_OK;
  if (!packed || !scales || !out || (need_zeros && !zeros)) {
    std::snprintf(msg, sizeof msg, "%s: null pointer", name);
    return int4lib::fail(INT4_ERR_ARG, msg);
  }
  const DType t = static_cast<DType>(out_dtype);
  if (!int4lib::aligned(out, int4lib::dtype_size(t)) || !int4lib::aligned(scales, 2)) {
    std::snprintf(msg, sizeof msg, "%s: out or scales not aligned to its element size", name);
    return int4lib::fail(INT4_ERR_ALIGN, msg);
  }
  const cudaError_t e = int4lib::launch_dequantize(packed, scales, need_zeros ? zeros : nullptr, K,
                                                   group, N, out, t, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, name);
}

int int4_dequantize_affine(const uint8_t* packed, const uint16_t* scales, const uint8_t* zeros,
                           int64_t K, int32_t group, int64_t N, void* out, int32_t out_dtype,
                           void* stream) {
  return dequantize_common("int4_dequantize_affine", packed, scales, zeros, true, K, group, N, out,
                           out_dtype, stream);
}

int int4_dequantize(const uint8_t* packed, const uint16_t* scales, int64_t K, int32_t group,
                    int64_t N, void* out, int32_t out_dtype, void* stream) {
  return dequantize_common("int4_dequantize", packed, scales, nullptr, false, K, group, N, out,
                           out_dtype, stream);
}

static int matmul_check(const void* x, int32_t x_dtype, const uint8_t* packed,
                        const uint16_t* scales, int64_t K, int32_t group, int64_t M, int64_t N,
                        const float* y) {
  if (!int4lib::dtype_ok(x_dtype)) return int4lib::fail(INT4_ERR_DTYPE, "int4_matmul: unknown x_dtype");
  if (M < 0 || N < 0 || K < 1 || group < 1)
    return int4lib::fail(INT4_ERR_ARG, "int4_matmul: need M, N >= 0, K >= 1, group >= 1");
  if (!int4lib::mul_ok(M, K) || !int4lib::mul_ok(N, K) || !int4lib::mul_ok(M, N))
    return int4lib::fail(INT4_ERR_ARG, "int4_matmul: sizes too large");
  if (M == 0 || N == 0) return INT4_OK;
  if (!x || !packed || !scales || !y) return int4lib::fail(INT4_ERR_ARG, "int4_matmul: null pointer");
  const DType t = static_cast<DType>(x_dtype);
  if (!int4lib::aligned(x, int4lib::dtype_size(t)) || !int4lib::aligned(scales, 2) ||
      !int4lib::aligned(y, 4))
    return int4lib::fail(INT4_ERR_ALIGN, "int4_matmul: x, scales or y not aligned to its element size");
  return INT4_OK;
}

static int matmul_choose(DType t, int64_t K, int32_t group, int64_t M, int64_t N, const void* x,
                         const uint8_t* packed) {
  if (int4lib::decode_supported(t, K, group, M, N, x, packed)) return INT4_PATH_DECODE;
  if (M > 16 && int4lib::prefill_supported(t, K, group, M, N, x, packed)) return INT4_PATH_PREFILL;
  return INT4_PATH_SIMT;
}

int int4_matmul_ex(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                   const uint8_t* zeros, int64_t K, int32_t group, int64_t M, int64_t N,
                   const float* bias, int32_t flags, float* y, int32_t path, void* workspace,
                   size_t workspace_bytes, void* stream) {
  const int rc = matmul_check(x, x_dtype, packed, scales, K, group, M, N, y);
  if (rc != INT4_OK || M == 0 || N == 0) return rc;
  if ((flags & ~INT4_EPI_RELU) != 0) return int4lib::fail(INT4_ERR_ARG, "int4_matmul: unknown flags");
  if (bias != nullptr && !int4lib::aligned(bias, 4))
    return int4lib::fail(INT4_ERR_ALIGN, "int4_matmul: bias not 4-byte aligned");
  if (workspace == nullptr && workspace_bytes != 0)
    return int4lib::fail(INT4_ERR_ARG, "int4_matmul: null workspace with a non-zero size");
  if (!int4lib::aligned(workspace, 256))
    return int4lib::fail(INT4_ERR_ALIGN, "int4_matmul: workspace not 256-byte aligned");
  const DType t = static_cast<DType>(x_dtype);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int4lib::Epilogue ep;
  ep.bias = bias;
  ep.relu = (flags & INT4_EPI_RELU) ? 1 : 0;
  if (path == INT4_PATH_AUTO) path = matmul_choose(t, K, group, M, N, x, packed);
  cudaError_t e;
  switch (path) {
    case INT4_PATH_SIMT:
      e = int4lib::launch_matmul_simt(x, t, packed, scales, zeros, K, group, M, N, ep, y, s);
      break;
    case INT4_PATH_DECODE: {
      if (!int4lib::decode_supported(t, K, group, M, N, x, packed))
        return int4lib::fail(INT4_ERR_UNSUPPORTED, "int4_matmul: decode kernel cannot run this shape");
      size_t need = 0;
      e = int4lib::launch_matmul_decode(x, t, packed, scales, zeros, ep, K, group, M, N, y,
                                        workspace, workspace_bytes, s, &need);
      if (e == cudaErrorInvalidValue && need > 0) {
        char msg[200];
        std::snprintf(msg, sizeof msg,
                      "int4_matmul: this call needs a workspace of %zu bytes, %zu given "
                      "(int4_matmul_workspace_size)",
                      need, workspace_bytes);
        return int4lib::fail(INT4_ERR_ARG, msg);
      }
      break;
    }
    case INT4_PATH_PREFILL:
      if (!int4lib::prefill_supported(t, K, group, M, N, x, packed))
        return int4lib::fail(INT4_ERR_UNSUPPORTED, "int4_matmul: tensor-core kernel cannot run this shape");
      e = int4lib::launch_matmul_prefill(x, t, packed, scales, zeros, ep, K, group, M, N, y,
                                         workspace, workspace_bytes, s);
      break;
    default:
      return int4lib::fail(INT4_ERR_ARG, "int4_matmul: unknown path");
  }
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_matmul");
}

int int4_matmul_path(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                     int64_t K, int32_t group, int64_t M, int64_t N, float* y, int32_t path,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return int4_matmul_ex(x, x_dtype, packed, scales, nullptr, K, group, M, N, nullptr, 0, y, path,
                        workspace, workspace_bytes, stream);
}

int int4_matmul(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                int64_t K, int32_t group, int64_t M, int64_t N, float* y, void* stream) {
  return int4_matmul_path(x, x_dtype, packed, scales, K, group, M, N, y, INT4_PATH_AUTO, nullptr, 0,
                          stream);
}

int int4_matmul_ws(const void* x, int32_t x_dtype, const uint8_t* packed, const uint16_t* scales,
                   int64_t K, int32_t group, int64_t M, int64_t N, float* y, void* workspace,
                   size_t workspace_bytes, void* stream) {
  return int4_matmul_path(x, x_dtype, packed, scales, K, group, M, N, y, INT4_PATH_AUTO, workspace,
                          workspace_bytes, stream);
}

int int4_matmul_workspace_size(int32_t x_dtype, int64_t K, int32_t group, int64_t M, int64_t N,
                               size_t* bytes) {
  if (bytes == nullptr) return int4lib::fail(INT4_ERR_ARG, "int4_matmul_workspace_size: null output");
  *bytes = 0;
  if (!int4lib::dtype_ok(x_dtype))
    return int4lib::fail(INT4_ERR_DTYPE, "int4_matmul_workspace_size: unknown x_dtype");
  if (M < 0 || N < 0 || K < 1 || group < 1)
    return int4lib::fail(INT4_ERR_ARG, "int4_matmul_workspace_size: need M, N >= 0, K >= 1, group >= 1");
  if (!int4lib::mul_ok(M, K) || !int4lib::mul_ok(N, K) || !int4lib::mul_ok(M, N))
    return int4lib::fail(INT4_ERR_ARG, "int4_matmul_workspace_size: sizes too large");
  if (M == 0 || N == 0) return INT4_OK;
  const DType t = static_cast<DType>(x_dtype);
  static const uint8_t* const kAligned = reinterpret_cast<const uint8_t*>(static_cast<uintptr_t>(256));
  const int path = matmul_choose(t, K, group, M, N, kAligned, kAligned);
  if (path == INT4_PATH_PREFILL) {
    // Non-zero only when the split of K pays (fewer tiles than SMs).
    *bytes = int4lib::prefill_workspace_size(K, group, M, N);
    return INT4_OK;
  }
  if (path != INT4_PATH_DECODE) return INT4_OK;
  const cudaError_t e = int4lib::decode_workspace_size(t, K, group, M, N, bytes);
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_matmul_workspace_size");
}

int int4_matmul_decode_noalloc(const void* x, int32_t x_dtype, const uint8_t* packed,
                               const uint16_t* scales, int64_t K, int32_t group, int64_t M,
                               int64_t N, float* y, void* stream) {
  const int rc = matmul_check(x, x_dtype, packed, scales, K, group, M, N, y);
  if (rc != INT4_OK || M == 0 || N == 0) return rc;
  const DType t = static_cast<DType>(x_dtype);
  if (!int4lib::decode_supported(t, K, group, M, N, x, packed))
    return int4lib::fail(INT4_ERR_UNSUPPORTED,
                         "int4_matmul_decode_noalloc: the decode kernel cannot run this shape "
                         "(needs bf16/fp16 x, M <= 16, K % 32 == 0, group 32, 64 or a multiple of "
                         "128, 16-byte aligned x and packed)");
  size_t need = 0;
  const cudaError_t e = int4lib::launch_matmul_decode_noalloc(
      x, t, packed, scales, K, group, M, N, y, static_cast<cudaStream_t>(stream), &need);
  if (e == cudaErrorInvalidValue && need > 0) {
    char msg[200];
    std::snprintf(msg, sizeof msg,
                  "int4_matmul_decode_noalloc: this call needs %zu bytes of scratch, the static "
                  "scratch holds %zu",
                  need, int4lib::decode_noalloc_scratch_bytes());
    return int4lib::fail(INT4_ERR_ARG, msg);
  }
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_matmul_decode_noalloc");
}

int int4_matmul_select(int32_t x_dtype, int64_t K, int32_t group, int64_t M, int64_t N) {
  if (!int4lib::dtype_ok(x_dtype)) return -INT4_ERR_DTYPE;
  if (M < 0 || N < 0 || K < 1 || group < 1) return -INT4_ERR_ARG;
  // Alignment of real buffers is not known here; assume allocator alignment.
  static const uint8_t* const kAligned = reinterpret_cast<const uint8_t*>(static_cast<uintptr_t>(256));
  return matmul_choose(static_cast<DType>(x_dtype), K, group, M, N, kAligned, kAligned);
}

int int4_device_status(void* stream) {
  uint32_t st = 0;
  const cudaError_t e = int4lib::read_and_clear_status(&st, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return int4lib::fail_cuda(e, "int4_device_status");
  if (st & int4lib::kStatusTimeout)
    return int4lib::fail(INT4_ERR_TIMEOUT, "a device-side bounded wait gave up");
  return INT4_OK;
}

int int4_selftest_wait_timeout(uint32_t spins, void* stream) {
  const cudaError_t e = int4lib::launch_wait_timeout_selftest(spins, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INT4_OK : int4lib::fail_cuda(e, "int4_selftest_wait_timeout");
}

}  // extern "C"
