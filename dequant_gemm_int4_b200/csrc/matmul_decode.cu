// Skinny dequantizing matmul for decode (M <= 16), sm_100a.
//
// y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * q[n, k]): the order of
// int4_matmul on the page "Implement INT4 group quantization, nibble packing
// and a dequantizing matmul" (problem statement), integer weights times x
// first, then the group's scale per output column.
//
// The kernel is bound by HBM: every packed weight byte is read once, and at
// M <= 16 each byte feeds at most 32 multiply-adds.  The design keeps the
// dequantization in registers:
//   * a warp owns 16 weight rows; each lane streams its share of every
//     128-wide K block with 16-byte (or, for group 64/32, 8/4-byte) loads
//     straight from HBM into registers;
//   * nibbles are sign-extended to bf16/fp16 with two integer ops per pair
//     ((w >> 4i) & 0x000F000F) ^ magic, then one packed subtract: the
//     magic 0x4300 / 0x6400 makes 128 + u (bf16) or 1024 + u (fp16) exactly,
//     u = q + 8, so every integer weight is exact;
//   * the 16 x 8 x 16 warp MMA (mma.sync, fp32 accumulate) multiplies them by
//     x, which sits in shared memory already permuted into fragment order, so
//     no multiply-add runs on the CUDA cores;
//   * each K group gets its own fp32 accumulator; its scale is applied with
//     one FMA per output into the fp32 running sum, per the page's order.
// Within one MMA the 16 k-slots of the four lanes of a quad are a
// permutation of the natural k order (pairs (e_i, e_{i+4}) of a 32-bit word);
// x is staged with the same permutation, and every MMA only sees k of one
// group.
// Split-K: when N is small the K range is split over the CTAs of a thread
// block cluster (up to 8); partial sums are reduced in a fixed order through
// distributed shared memory, so the result is deterministic and the kernel
// needs no memory beyond its inputs and outputs.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace int4lib {

namespace {

constexpr int kWarps = 8;                 // warps per CTA, one 16-row tile each
constexpr int kRowsPerCta = 16 * kWarps;  // 128 weight rows per CTA
constexpr int kPrefetch = 4;              // K blocks loaded ahead per warp
constexpr int kChunkBlocks = 16;          // K blocks of x staged per pass
constexpr int kMaxCluster = 8;

template <typename TX>
struct Cvt;
// bf16: (w & 0x000F000F) ^ 0x43084308 = bf16x2(128 + u_lo, 128 + u_hi), u = q + 8.
template <>
struct Cvt<__nv_bfloat16> {
  static constexpr uint32_t kMagic = 0x43084308u;
  static constexpr uint32_t kBias = 0x43084308u;  // bf16x2(136, 136)
  __device__ __forceinline__ static uint32_t sub(uint32_t a) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(kBias));
    return d;
  }
  __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};
// fp16: (w & 0x000F000F) ^ 0x64086408 = f16x2(1024 + u_lo, 1024 + u_hi).
template <>
struct Cvt<__half> {
  static constexpr uint32_t kMagic = 0x64086408u;
  static constexpr uint32_t kBias = 0x64086408u;  // f16x2(1032, 1032)
  __device__ __forceinline__ static uint32_t sub(uint32_t a) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(kBias));
    return d;
  }
  __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};

// Word w holds nibbles e0..e7 (k = 8*widx + 0..7).  p[i] = (e_i, e_{i+4}).
template <typename TX>
__device__ __forceinline__ void expand(uint32_t w, uint32_t (&p)[4]) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x000F000Fu), "r"(Cvt<TX>::kMagic));
  p[0] = Cvt<TX>::sub(t);
#pragma unroll
  for (int i = 1; i < 4; ++i) {
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;"
        : "=r"(t)
        : "r"(w >> (4 * i)), "r"(0x000F000Fu), "r"(Cvt<TX>::kMagic));
    p[i] = Cvt<TX>::sub(t);
  }
}

// Which 8-k group (0..15 inside a 128-k block) lane c uses as its word j,
// for GPB groups per block (1: group >= 128, 2: group 64, 4: group 32), so
// that all four lanes of a quad read the same group for word j.
template <int GPB>
__device__ __forceinline__ int word_index(int c, int j) {
  if (GPB == 1) return 4 * c + j;
  if (GPB == 2) return (j >> 1) * 8 + 2 * c + (j & 1);
  return 4 * j + c;
}

template <int GPB>
__device__ __forceinline__ void word_owner(int kk, int& c, int& j) {
  if (GPB == 1) {
    c = kk >> 2;
    j = kk & 3;
  } else if (GPB == 2) {
    j = (kk >> 3) * 2 + (kk & 1);
    c = (kk & 7) >> 1;
  } else {
    j = kk >> 2;
    c = kk & 3;
  }
}

// Loads this lane's four words of one 128-k block of row `rowp` (row start).
template <int GPB>
__device__ __forceinline__ void load_words(const uint8_t* rowp, bool row_ok, int64_t kb, int c,
                                           int64_t K, uint32_t (&w)[4]) {
  const uint8_t* bp = rowp + kb * 64;
  const int64_t kbase = kb * 128;
  if (GPB == 1) {
    if (row_ok && kbase + 32 * c < K) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(bp + 16 * c));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
      w[0] = w[1] = w[2] = w[3] = 0x88888888u & 0u;
    }
  } else if (GPB == 2) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (row_ok && kbase + 64 * h + 16 * c < K) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(bp + 32 * h + 8 * c));
        w[2 * h] = v.x; w[2 * h + 1] = v.y;
      } else {
        w[2 * h] = w[2 * h + 1] = 0u;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[j] = (row_ok && kbase + 32 * j + 8 * c < K)
                 ? __ldg(reinterpret_cast<const uint32_t*>(bp + 16 * j + 4 * c))
                 : 0u;
    }
  }
}

// Shared memory: x chunk in fragment order, then the split-K partials.
//   xs[((kbl * 4 + j) * NT + nt) * 32 + lane] : uint4 = 8 x values of
//   batch row nt*8 + lane/4, k8-group word_index(lane%4, j) of block kbl,
//   as (x0,x4) (x1,x5) (x2,x6) (x3,x7).
template <typename TX, int NT, int GPB>
__global__ void __launch_bounds__(256, 2) decode_kernel(
    const TX* __restrict__ x, const uint8_t* __restrict__ packed,
    const uint16_t* __restrict__ scales, int64_t K, int group, int G, int M, int64_t N,
    float* __restrict__ y, int kblocks_per_slice, int S) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint4* xs = reinterpret_cast<uint4*>(smem);
  float* red = reinterpret_cast<float*>(smem + kChunkBlocks * 16 * NT * 8 * 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = lane & 3;
  const int g = lane >> 2;
  const int slice = blockIdx.x;  // == rank in the cluster when S > 1
  const int64_t KB = (K + 127) / 128;
  const int64_t kb0 = static_cast<int64_t>(slice) * kblocks_per_slice;
  int64_t kb1 = kb0 + kblocks_per_slice;
  if (kb1 > KB) kb1 = KB;
  const int64_t Kp = K >> 1;
  const int64_t ra = static_cast<int64_t>(blockIdx.y) * kRowsPerCta + warp * 16 + g;
  const int64_t rb = ra + 8;
  const bool va = ra < N, vb = rb < N;
  const uint8_t* rowa = packed + (va ? ra : 0) * Kp;
  const uint8_t* rowb = packed + (vb ? rb : 0) * Kp;

  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) tot[nt][i] = 0.0f;

  for (int64_t cb0 = kb0; cb0 < kb1; cb0 += kChunkBlocks) {
    const int64_t cb1 = (cb0 + kChunkBlocks < kb1) ? cb0 + kChunkBlocks : kb1;
    const int nblk = static_cast<int>(cb1 - cb0);
    // Stage x[:, cb0*128 : cb1*128] in fragment order (zeros past M and K).
    __syncthreads();
    const int entries = nblk * 16 * NT * 8;
    for (int e = threadIdx.x; e < entries; e += blockDim.x) {
      const int m = e % (NT * 8);
      const int kk = (e / (NT * 8)) % 16;
      const int kbl = e / (NT * 8 * 16);
      const int64_t k = (cb0 + kbl) * 128 + kk * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (m < M && k < K) {
        const uint4 r = __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k));
        v.x = __byte_perm(r.x, r.z, 0x5410);
        v.y = __byte_perm(r.x, r.z, 0x7632);
        v.z = __byte_perm(r.y, r.w, 0x5410);
        v.w = __byte_perm(r.y, r.w, 0x7632);
      }
      int cc, jj;
      word_owner<GPB>(kk, cc, jj);
      xs[((kbl * 4 + jj) * NT + (m >> 3)) * 32 + (m & 7) * 4 + cc] = v;
    }
    __syncthreads();

    for (int64_t kb = cb0; kb < cb1; kb += kPrefetch) {
      uint32_t wa[kPrefetch][4], wb[kPrefetch][4];
#pragma unroll
      for (int p = 0; p < kPrefetch; ++p) {
        if (kb + p < cb1) {
          load_words<GPB>(rowa, va, kb + p, c, K, wa[p]);
          load_words<GPB>(rowb, vb, kb + p, c, K, wb[p]);
        }
      }
#pragma unroll
      for (int p = 0; p < kPrefetch; ++p) {
        if (kb + p >= cb1) break;
        const int kbl = static_cast<int>(kb + p - cb0);
        float acc[GPB][NT][4];
#pragma unroll
        for (int a = 0; a < GPB; ++a)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[a][nt][i] = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pa[4], pb[4];
          expand<TX>(wa[p][j], pa);
          expand<TX>(wb[p][j], pb);
          const int a = (GPB == 1) ? 0 : (GPB == 2 ? (j >> 1) : j);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint4 xf = xs[((kbl * 4 + j) * NT + nt) * 32 + lane];
            Cvt<TX>::mma(acc[a][nt], pa[0], pb[0], pa[1], pb[1], xf.x, xf.y);
            Cvt<TX>::mma(acc[a][nt], pa[2], pb[2], pa[3], pb[3], xf.z, xf.w);
          }
        }
        // Apply each group's scale per output row, then add to the running sum.
        const int64_t kbase = (kb + p) * 128;
#pragma unroll
        for (int a = 0; a < GPB; ++a) {
          const int64_t gi = (kbase + a * (128 / GPB)) / group;
          const float sa = (va && gi < G) ? f16_bits_to_float(__ldg(scales + ra * G + gi)) : 0.0f;
          const float sb = (vb && gi < G) ? f16_bits_to_float(__ldg(scales + rb * G + gi)) : 0.0f;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            tot[nt][0] = fmaf(acc[a][nt][0], sa, tot[nt][0]);
            tot[nt][1] = fmaf(acc[a][nt][1], sa, tot[nt][1]);
            tot[nt][2] = fmaf(acc[a][nt][2], sb, tot[nt][2]);
            tot[nt][3] = fmaf(acc[a][nt][3], sb, tot[nt][3]);
          }
        }
      }
    }
  }

  // Output (m, row) of register i of n-tile nt: m = nt*8 + 2c + (i & 1),
  // row = (i < 2) ? ra : rb.
  if (S == 1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = nt * 8 + 2 * c + (i & 1);
        const int64_t row = (i < 2) ? ra : rb;
        if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = tot[nt][i];
      }
    return;
  }

  // Split-K: partials to shared memory, reduce across the cluster in rank order.
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[((warp * NT + nt) * 4 + i) * 32 + lane] = tot[nt][i];
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  const int total = kWarps * NT * 4 * 32;
  for (int e = slice * blockDim.x + threadIdx.x; e < total; e += S * blockDim.x) {
    float s = 0.0f;
    for (int r = 0; r < S; ++r) s += cluster.map_shared_rank(red, r)[e];
    const int ln = e & 31;
    const int i = (e >> 5) & 3;
    const int nt = (e >> 7) % NT;
    const int wp = (e >> 7) / NT;
    const int m = nt * 8 + 2 * (ln & 3) + (i & 1);
    const int64_t row = static_cast<int64_t>(blockIdx.y) * kRowsPerCta + wp * 16 + (ln >> 2) +
                        ((i < 2) ? 0 : 8);
    if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = s;
  }
  cluster.sync();  // keep this CTA's partials alive until every rank has read them
}

template <typename TX, int NT, int GPB>
cudaError_t launch_variant(const TX* x, const uint8_t* packed, const uint16_t* scales, int64_t K,
                           int group, int64_t M, int64_t N, float* y, cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const int64_t KB = (K + 127) / 128;
  const int64_t R = (N + kRowsPerCta - 1) / kRowsPerCta;
  if (R > 65535) return cudaErrorInvalidConfiguration;
  // Enough CTAs to cover the SMs about twice; at most 8 K slices.
  const int64_t target = 2LL * num_sms();
  int64_t S = (target + R - 1) / R;
  if (S > kMaxCluster) S = kMaxCluster;
  if (S > KB) S = KB;
  if (S < 1) S = 1;
  const int kbps = static_cast<int>((KB + S - 1) / S);
  S = (KB + kbps - 1) / kbps;  // no empty slices
  const size_t smem = static_cast<size_t>(kChunkBlocks) * 16 * NT * 8 * 16 +
                      static_cast<size_t>(kWarps) * NT * 4 * 32 * sizeof(float);
  auto kern = decode_kernel<TX, NT, GPB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S), static_cast<unsigned>(R), 1);
  cfg.blockDim = dim3(32 * kWarps, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, packed, scales, K, group, G, static_cast<int>(M), N, y,
                            kbps, static_cast<int>(S));
}

template <typename TX, int NT>
cudaError_t launch_nt(const TX* x, const uint8_t* packed, const uint16_t* scales, int64_t K,
                      int group, int64_t M, int64_t N, float* y, cudaStream_t stream) {
  if (group % 128 == 0) return launch_variant<TX, NT, 1>(x, packed, scales, K, group, M, N, y, stream);
  if (group == 64) return launch_variant<TX, NT, 2>(x, packed, scales, K, group, M, N, y, stream);
  return launch_variant<TX, NT, 4>(x, packed, scales, K, group, M, N, y, stream);
}

template <typename TX>
cudaError_t launch_tx(const TX* x, const uint8_t* packed, const uint16_t* scales, int64_t K,
                      int group, int64_t M, int64_t N, float* y, cudaStream_t stream) {
  if (M <= 8) return launch_nt<TX, 1>(x, packed, scales, K, group, M, N, y, stream);
  return launch_nt<TX, 2>(x, packed, scales, K, group, M, N, y, stream);
}

}  // namespace

bool decode_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                      const uint8_t* packed) {
  if (xt == DType::F32) return false;
  if (M < 1 || M > 16 || N < 1) return false;
  if (K % 32 != 0) return false;
  if (!(group == 32 || group == 64 || group % 128 == 0)) return false;
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0) return false;
  if (reinterpret_cast<uintptr_t>(packed) % 16 != 0) return false;
  if ((N + kRowsPerCta - 1) / kRowsPerCta > 65535) return false;
  return true;
}

cudaError_t launch_matmul_decode(const void* x, DType xt, const uint8_t* packed,
                                 const uint16_t* scales, int64_t K, int group, int64_t M,
                                 int64_t N, float* y, cudaStream_t stream) {
  if (xt == DType::BF16)
    return launch_tx(static_cast<const __nv_bfloat16*>(x), packed, scales, K, group, M, N, y,
                     stream);
  return launch_tx(static_cast<const __half*>(x), packed, scales, K, group, M, N, y, stream);
}

}  // namespace int4lib
