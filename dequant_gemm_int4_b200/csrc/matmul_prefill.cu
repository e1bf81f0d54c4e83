// Tensor-core dequantizing matmul for large M (prefill), sm_100a.
//
// y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * q[n, k]): int4_matmul of
// the page "Implement INT4 group quantization, nibble packing and a
// dequantizing matmul" (problem statement), computed one K group at a time
// with the group's scale applied to each output before the fp32 running sum.
//
// One CTA computes a 128 (weight rows n) x BM (activation rows m) tile of y^T
// with tcgen05 MMAs (kind::f16, fp32 accumulation in tensor memory):
//   warp 0      TMA producer: per 64-wide K stage, the packed weights
//               [128 rows x 32 bytes] and x [BM rows x 64] (128-byte swizzle)
//   warps 4-7   dequantizers: thread t expands weight row t of the stage from
//               nibbles to bf16/fp16 (exact: 128 + u or 1024 + u minus 136 or
//               1032) into the A tile, K-major with the 128-byte swizzle
//   warp 1      MMA issuer: D_g = A_g * X_g^T into one of two TMEM partial
//               buffers (128 lanes x BM columns), one buffer per K group
//   warps 8-15  epilogue: for every group, load the group's partial from TMEM,
//               multiply by s[n, g] (one scale per TMEM lane = weight row) and
//               add into fp32 registers; finally store y.
// TMEM lane = weight row n, so the per-(column, group) scale of the page is a
// single register per thread.  Stages flow through full/empty mbarriers; the
// two TMEM partial buffers let the tensor core run group g+1 while the
// epilogue drains group g.  Every wait is bounded in time: a wait that gives
// up sets an abort flag and the status word, every role leaves its loop,
// outstanding copies and MMAs are drained (again with a bound) and TMEM is
// freed before the CTA exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace int4lib {

namespace {

constexpr int kBN = 128;      // weight rows per tile (MMA M)
constexpr int kKS = 64;       // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 512;
// Raster: the grid walks runs of kGroupM activation-row tiles, all weight-row
// tiles of a run before the next (activation tile fastest).  A run's x tiles
// (8 x 4 MB at K = 8192) stay in L2 while the weight tiles stream past, and
// each weight tile is read once per run instead of once per x tile.
#ifndef INT4_PREFILL_GROUP_M
#define INT4_PREFILL_GROUP_M 8
#endif
constexpr int kGroupM = INT4_PREFILL_GROUP_M;
constexpr uint64_t kTimeoutNs = 250000000ull;  // 250 ms: far above any legitimate wait

struct Barriers {
  uint64_t full_tma[kStages];   // TMA bytes of stage s landed
  uint64_t full_a[kStages];     // dequantized A tile of stage s written
  uint64_t empty[kStages];      // MMAs reading stage s finished
  uint64_t tmem_full[2];        // group partial in TMEM buffer b complete
  uint64_t tmem_empty[2];       // epilogue finished reading buffer b
  uint64_t drain;               // abort path: all issued MMAs finished
};

template <int BM>
struct Layout {
  static constexpr int kA = kBN * kKS * 2;  // 16 KB
  static constexpr int kX = BM * kKS * 2;   // 32 KB at BM = 256
  static constexpr int kP = kBN * kKS / 2;  // 4 KB
  static constexpr int offA = 0;
  static constexpr int offX = offA + kStages * kA;
  static constexpr int offP = offX + kStages * kX;
  static constexpr int offBar = offP + kStages * kP;
  static constexpr int offMisc = offBar + static_cast<int>(sizeof(Barriers));
  static constexpr int kBytes = offMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 2 * BM;
};

// Instruction descriptor, kind::f16: D fp32, A/B bf16 (1) or fp16 (0),
// both K-major, N = BM, M = 128.
template <typename TX, int BM>
__device__ __forceinline__ constexpr uint32_t make_idesc() {
  constexpr uint32_t ab = std::is_same<TX, __nv_bfloat16>::value ? 1u : 0u;
  return (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(BM >> 3) << 17) |
         (static_cast<uint32_t>(kBN >> 4) << 24);
}

template <typename TX>
struct Nib;
template <>
struct Nib<__nv_bfloat16> {
  static constexpr uint32_t kMagic = 0x43084308u;  // bf16 128 in each half, nibble sign bit flipped
  static constexpr uint32_t kBase = 0x43004300u;   // bf16 128 in each half (unsigned codes)
  __device__ __forceinline__ static uint32_t zero_bias(uint32_t z) { return (0x4300u + z) * 0x00010001u; }
  __device__ __forceinline__ static uint32_t sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));  // - 136, or - (128 + z)
    return d;
  }
};
template <>
struct Nib<__half> {
  static constexpr uint32_t kMagic = 0x64086408u;  // fp16 1024 in each half
  static constexpr uint32_t kBase = 0x64006400u;
  __device__ __forceinline__ static uint32_t zero_bias(uint32_t z) { return (0x6400u + z) * 0x00010001u; }
  __device__ __forceinline__ static uint32_t sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));  // - 1032, or - (1024 + z)
    return d;
  }
};

// 4 packed bytes (8 consecutive k) -> 8 bf16/fp16 in natural k order: q
// (two's-complement nibbles), or q - z for unsigned codes (ASYM, zb =
// zero_bias(z)).
template <typename TX, bool ASYM>
__device__ __forceinline__ uint4 expand8(uint32_t w, uint32_t zb) {
  constexpr uint32_t kx = ASYM ? Nib<TX>::kBase : Nib<TX>::kMagic;
  const uint32_t ws = w >> 4;
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // byte j low nibble -> bits 0..3, byte j high nibble -> bits 16..19
    const uint32_t sel = static_cast<uint32_t>(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
    const uint32_t t = __byte_perm(w, ws, sel);
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(t), "r"(0x000F000Fu), "r"(kx));
    o[j] = Nib<TX>::sub(r, ASYM ? zb : Nib<TX>::kMagic);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

struct WaitCtx {
  volatile uint32_t* abort;
  uint32_t* status;
};

// Bounded wait on an mbarrier phase.  Returns false if the CTA is aborting or
// the wait exceeded the time limit (which starts the abort).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t i = 1; i != 0; ++i) {
    if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if ((i & 15u) == 0u) {
      if (*w.abort) return false;
      if (ptx::globaltimer() - t0 > kTimeoutNs) break;
    }
  }
  *w.abort = 1u;
  report_status(w.status, kStatusTimeout);
  return false;
}

// Bounded wait used only on the abort path (ignores the abort flag).
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t i = 0; i != 0xFFFFFFFFu; ++i) {
    if (ptx::mbar_try_wait(bar, parity)) return;
    if ((i & 127u) == 0u && ptx::globaltimer() - t0 > kTimeoutNs) return;
  }
}

template <typename TX, int BM, bool ASYM>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_p,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros, Epilogue ep,
    float* __restrict__ y, int M, int N, int K, int group, int G, uint32_t* status) {
  using L = Layout<BM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + L::offBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int n0, m0;
  {
    const int num_n = (N + kBN - 1) / kBN, num_m = (M + BM - 1) / BM;
    const int per_run = kGroupM * num_n;
    const int run = static_cast<int>(blockIdx.x) / per_run;
    const int first_m = run * kGroupM;
    const int gm = (num_m - first_m < kGroupM) ? num_m - first_m : kGroupM;
    const int r = static_cast<int>(blockIdx.x) - run * per_run;
    n0 = (r / gm) * kBN;
    m0 = (first_m + r % gm) * BM;
  }
  const int nstages = (K + kKS - 1) / kKS;

  const uint32_t sA = ptx::smem_u32(smem + L::offA);
  const uint32_t sX = ptx::smem_u32(smem + L::offX);
  const uint32_t sP = ptx::smem_u32(smem + L::offP);
  auto bar = [&](uint64_t* b) { return ptx::smem_u32(b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(&bars->full_tma[s]), 1);
      ptx::mbar_init(bar(&bars->full_a[s]), 128);
      ptx::mbar_init(bar(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(&bars->tmem_full[b]), 1);
      ptx::mbar_init(bar(&bars->tmem_empty[b]), 256);
    }
    ptx::mbar_init(bar(&bars->drain), 1);
    *abort_flag = 0u;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_x);
    ptx::prefetch_tmap(&tm_p);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), L::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const WaitCtx wc{abort_flag, status};

  if (warp < 4) {
    ptx::regs_dec<24>();
    if (warp == 0 && lane == 0) {
      // ---------------- TMA producer ----------------
      int it = 0;
      for (; it < nstages; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!wait_bar(bar(&bars->empty[s]), ph ^ 1u, wc)) break;
        ptx::mbar_arrive_expect_tx(bar(&bars->full_tma[s]), L::kX + L::kP);
        ptx::tma_load_2d(sX + s * L::kX, &tm_x, it * kKS, m0, bar(&bars->full_tma[s]));
        ptx::tma_load_2d(sP + s * L::kP, &tm_p, it * (kKS / 2), n0, bar(&bars->full_tma[s]));
      }
      if (*abort_flag) {
        // Let every issued copy land before the CTA's shared memory goes away.
        const int first = it - kStages > 0 ? it - kStages : 0;
        for (int j = first; j < it; ++j)
          drain_bar(bar(&bars->full_tma[j % kStages]), (j / kStages) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = make_idesc<TX, BM>();
      int gi = 0;
      for (int it = 0; it < nstages; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int k0 = it * kKS;
        const bool first_of_group = (k0 % group) == 0;
        const bool last_of_group = ((k0 + kKS) % group) == 0 || (k0 + kKS) >= K;
        const int buf = gi & 1;
        if (first_of_group) {
          if (!wait_bar(bar(&bars->tmem_empty[buf]), ((gi >> 1) & 1) ^ 1u, wc)) break;
          ptx::tc_fence_after();
        }
        if (!wait_bar(bar(&bars->full_tma[s]), ph, wc)) break;
        if (!wait_bar(bar(&bars->full_a[s]), ph, wc)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BM);
#pragma unroll
        for (int kk = 0; kk < kKS / 16; ++kk) {
          const uint64_t ad = ptx::sw128_kmajor_desc(sA + s * L::kA + kk * 32);
          const uint64_t bd = ptx::sw128_kmajor_desc(sX + s * L::kX + kk * 32);
          ptx::umma_f16(d, ad, bd, idesc, (first_of_group && kk == 0) ? 0u : 1u);
        }
        ptx::umma_commit(bar(&bars->empty[s]));
        if (last_of_group) {
          ptx::umma_commit(bar(&bars->tmem_full[buf]));
          ++gi;
        }
      }
      if (*abort_flag) {
        ptx::umma_commit(bar(&bars->drain));
        drain_bar(bar(&bars->drain), 0);
      }
    }
  } else if (warp < 8) {
    ptx::regs_dec<72>();
    // ---------------- dequantizers: thread t owns weight row t ----------------
    const int t = threadIdx.x - 128;
    const int swz = t & 7;
    const int first = (t >> 2) & 1;  // rotates the two 16-byte reads to avoid bank conflicts
    const uint8_t* zrow = ASYM ? zeros + static_cast<int64_t>(n0 + t < N ? n0 + t : N - 1) * G : nullptr;
    for (int it = 0; it < nstages; ++it) {
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      // The stage's zero point (a stage lies inside one group).
      const uint32_t zb = ASYM ? Nib<TX>::zero_bias(__ldg(zrow + (it * kKS) / group)) : 0u;
      if (!wait_bar(bar(&bars->full_tma[s]), ph, wc)) break;
      const uint32_t prow = sP + s * L::kP + t * 32;
      const uint4 va = ptx::lds128(prow + 16 * first);
      const uint4 vb = ptx::lds128(prow + 16 * (first ^ 1));
      const uint4 lo = first ? vb : va;
      const uint4 hi = first ? va : vb;
      const uint32_t wds[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
      const uint32_t arow = sA + s * L::kA + t * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) ptx::sts128(arow + ((c ^ swz) << 4), expand8<TX, ASYM>(wds[c], zb));
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(bar(&bars->full_a[s]));
    }
  } else {
    ptx::regs_inc<208>();
    // ---------------- epilogue: lane quarter q, column half h ----------------
    const int q = warp & 3;
    const int h = (warp - 8) >> 2;
    const int row = 32 * q + lane;
    const int n = n0 + row;
    constexpr int kCols = BM / 2;
    float acc[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) acc[j] = 0.0f;
    const uint16_t* srow = scales + static_cast<int64_t>(n < N ? n : 0) * G;
    float s_next = (n < N) ? f16_bits_to_float(__ldg(srow)) : 0.0f;
    bool ok = true;
    for (int gi = 0; gi < G; ++gi) {
      const int buf = gi & 1;
      const float sc = s_next;
      if (gi + 1 < G && n < N) s_next = f16_bits_to_float(__ldg(srow + gi + 1));
      if (!wait_bar(bar(&bars->tmem_full[buf]), (gi >> 1) & 1, wc)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                             static_cast<uint32_t>(buf * BM + h * kCols);
#pragma unroll
      for (int c = 0; c < kCols; c += 16) {
        uint32_t r[16];
        ptx::tmem_ld_32x32b_x16(taddr + c, r);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[c + j] = fmaf(__uint_as_float(r[j]), sc, acc[c + j]);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(&bars->tmem_empty[buf]));
    }
    if (ok && n < N) {
      const int mbase = m0 + h * kCols;
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        const int m = mbase + j;
        if (m < M) y[static_cast<int64_t>(m) * N + n] = ep.apply(acc[j], n);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <typename TX, int BM, bool ASYM>
cudaError_t launch_bm(const TX* x, const uint8_t* packed, const uint16_t* scales,
                      const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                      int64_t N, float* y, cudaStream_t stream) {
  using L = Layout<BM>;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  uint32_t* status = status_word();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  CUtensorMap tx, tp;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {kKS, BM};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = std::is_same<TX, __nv_bfloat16>::value
                                       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (enc(&tx, dt, 2, const_cast<TX*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int64_t Kp = K / 2;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kp), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kp)};
    const cuuint32_t box[2] = {kKS / 2, kBN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = prefill_kernel<TX, BM, ASYM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(((N + kBN - 1) / kBN) * ((M + BM - 1) / BM)));
  const int G = static_cast<int>((K + group - 1) / group);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(tx, tp, scales, zeros, ep, y, static_cast<int>(M),
                                              static_cast<int>(N), static_cast<int>(K), group, G,
                                              status);
  return cudaGetLastError();
}

}  // namespace

bool prefill_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                       const uint8_t* packed) {
  if (xt == DType::F32) return false;
  if (M < 1 || N < 1 || K < 1) return false;
  if (K % 32 != 0 || group % kKS != 0) return false;
  if (K > (1LL << 30) || M > (1LL << 30) || N > (1LL << 30)) return false;
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0 || reinterpret_cast<uintptr_t>(packed) % 16 != 0)
    return false;
  if (((N + kBN - 1) / kBN) * ((M + 255) / 256) > 0x7FFFFFFFLL) return false;
  return true;
}

template <typename TX>
static cudaError_t launch_prefill_tx(const TX* x, const uint8_t* packed, const uint16_t* scales,
                                     const uint8_t* zeros, const Epilogue& ep, int64_t K, int group,
                                     int64_t M, int64_t N, float* y, cudaStream_t stream) {
  if (zeros != nullptr)
    return launch_bm<TX, 256, true>(x, packed, scales, zeros, ep, K, group, M, N, y, stream);
  return launch_bm<TX, 256, false>(x, packed, scales, nullptr, ep, K, group, M, N, y, stream);
}

cudaError_t launch_matmul_prefill(const void* x, DType xt, const uint8_t* packed,
                                  const uint16_t* scales, const uint8_t* zeros, const Epilogue& ep,
                                  int64_t K, int group, int64_t M, int64_t N, float* y,
                                  cudaStream_t stream) {
  if (xt == DType::BF16)
    return launch_prefill_tx(static_cast<const __nv_bfloat16*>(x), packed, scales, zeros, ep, K,
                             group, M, N, y, stream);
  return launch_prefill_tx(static_cast<const __half*>(x), packed, scales, zeros, ep, K, group, M, N,
                           y, stream);
}

}  // namespace int4lib
