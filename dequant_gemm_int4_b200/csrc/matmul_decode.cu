// Skinny dequantizing matmul for decode (M <= 16), sm_100a.
//
// y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * q[n, k]): the order of
// int4_matmul on the page "Implement INT4 group quantization, nibble packing
// and a dequantizing matmul" (problem statement), integer weights times x
// first, then the group's scale per output column.
//
// Two kernels share the CTA structure below.  For a group that is a multiple
// of 128 (the common case) decode_i8_kernel runs the products on the int8
// warp MMA, with x split into base-256 digits (its comment block gives the
// arithmetic); for groups of 32 and 64, decode_kernel expands nibbles to
// bf16/fp16 and runs the 16-bit warp MMA, as described here.
//
// The kernel is bound by HBM: every packed weight byte is read once and at
// M <= 16 feeds at most 32 multiply-adds.  Design:
//   * a producer warp streams 128 weight rows (64 for M > 8) through a
//     3-stage shared-memory ring with TMA (each stage: the rows x 256 k of
//     packed nibbles, 128-byte swizzle, plus x [M x 256] bf16/fp16), two CTAs
//     per SM;
//   * eight consumer warps, four row groups x two K-block slots per stage;
//     a row group is 32 rows (two 16-row tiles) so every x fragment feeds two
//     independent MMA chains; per 128-wide K block a lane reads its 16 (or
//     2 x 8, 4 x 4 for group 64/32) bytes of four rows from shared memory and
//     sign-extends nibble pairs to bf16/fp16 exactly in
//     registers: for a 32-bit word of nibbles e0..e7, the pair (e_i, e_{i+4})
//     is ((w >> 4i) & 0x000F000F) ^ magic, then one packed subtract (magic =
//     128 + 8 (bf16) or 1024 + 8 (fp16) in each half; the XOR flips the
//     nibble's sign bit so that the value is q + 136 or q + 1032 before the
//     subtract);
//   * the 16 x 8 x 16 warp MMA (mma.sync, fp32 accumulate) multiplies them by
//     x from shared memory; the MMA's k slots see the pairs (e_i, e_{i+4}), so
//     x is paired the same way in registers (four byte permutes per 16 bytes,
//     shared by the warp's two row tiles), and no multiply-add runs on the
//     CUDA cores;
//   * each K group gets its own fp32 accumulator, which is scaled by its
//     group's scale and added into the fp32 running sum, per the page's order.
// Lanes of padding batch rows (n >= M) use zero x fragments and skip their
// shared-memory loads.  All four lanes of a quad read the same group for a
// given word, so each MMA only sums k of one group.  Weight rows are permuted
// inside each 16-row tile so that the shared-memory loads are free of bank
// conflicts.
//
// Work split (stream-K): the (row tile, 128-k block) units are dealt out in
// row-major order as equal contiguous runs to one wave of CTAs (two per SM),
// so every SM streams the same number of bytes whatever N and K are.  A tile
// that a run covers whole is written to y by its CTA; each piece of a tile
// that straddles runs goes to a partial slot, its CTA counts its arrival, and
// the last contributor to arrive adds the pieces in CTA order (so the result
// does not depend on timing), writes y and resets the count.  Every mbarrier
// wait is bounded in time; a wait that gives up aborts the CTA (the status
// word records it), drains its copies and skips the output.
#include <cuda.h>

#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace int4lib {

namespace {

// Shape of a CTA (compile-time; the defaults are the measured choice).
#ifndef INT4_DECODE_SK
#define INT4_DECODE_SK 2
#endif
#ifndef INT4_DECODE_ROW_GROUPS
#define INT4_DECODE_ROW_GROUPS 4
#endif
#ifndef INT4_DECODE_STAGES
#define INT4_DECODE_STAGES 3
#endif
#ifndef INT4_DECODE_TILES1
#define INT4_DECODE_TILES1 2
#endif
#ifndef INT4_DECODE_MIN_BLOCKS
#define INT4_DECODE_MIN_BLOCKS 2
#endif
#ifndef INT4_DECODE_I8_MINB1
#define INT4_DECODE_I8_MINB1 2
#endif
#ifndef INT4_DECODE_I8_FUSE_MAX_M
#define INT4_DECODE_I8_FUSE_MAX_M 2
#endif
#ifndef INT4_DECODE_WAIT_MODE
#define INT4_DECODE_WAIT_MODE 0  // 0: try_wait, then 20 us suspend hints; 1: test_wait polling; 2: 500 ns hints
#endif
#ifndef INT4_DECODE_SMALL
#define INT4_DECODE_SMALL 1
#endif
#ifndef INT4_DECODE_FLAT
#define INT4_DECODE_FLAT 1
#endif
#ifndef INT4_DECODE_I8_TILES
#define INT4_DECODE_I8_TILES 2
#endif
#ifndef INT4_DECODE_I8_SCALE_AHEAD
#define INT4_DECODE_I8_SCALE_AHEAD 1
#endif
#ifndef INT4_DECODE_L2_AHEAD
#define INT4_DECODE_L2_AHEAD 0  // integer kernel: stages beyond the ring whose weights are prefetched into L2
#endif
constexpr int kSK = INT4_DECODE_SK;                // 128-wide K blocks per stage (even)
constexpr int kFuseMaxM = INT4_DECODE_I8_FUSE_MAX_M;  // batch rows the in-kernel x conversion serves
constexpr int kSub = kSK / 2;                      // 256-k sub-tiles per stage (one copy each)
static_assert(kSK % 2 == 0, "stages hold whole 256-k sub-tiles");
constexpr int kRowGroups = INT4_DECODE_ROW_GROUPS;  // row groups per CTA
constexpr int kConsumers = kRowGroups * kSK;  // one consumer warp per (row group, block of the stage)
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = INT4_DECODE_STAGES;

// 16-row tiles per consumer warp: two for M <= 8 (NT = 1), one for M <= 16,
// so that both fit two CTAs per SM without spilling.
template <int NT>
struct Tiles {
  static constexpr int kTiles = NT == 1 ? INT4_DECODE_TILES1 : 1;
  static constexpr int kRowsPerCta = 16 * kTiles * kRowGroups;  // 128 or 64
  static constexpr int kWBytes = kRowsPerCta * kSK * 64;          // 16 or 8 KB per stage
};
constexpr uint64_t kTimeoutNs = 250000000ull;

template <typename TX>
struct Cvt;
template <>
struct Cvt<__nv_bfloat16> {
  static constexpr uint32_t kMagic = 0x43084308u;  // 128 + 8 in each half (the XOR flips the sign bit)
  static constexpr uint32_t kBase = 0x43004300u;   // 128 in each half (unsigned codes)
  // The subtrahend for unsigned codes with zero point z: 128 + z in each half.
  __device__ __forceinline__ static uint32_t zero_bias(uint32_t z) { return (0x4300u + z) * 0x00010001u; }
  __device__ __forceinline__ static uint32_t sub(uint32_t a, uint32_t b = 0x43084308u) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
  }
  __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};
template <>
struct Cvt<__half> {
  static constexpr uint32_t kMagic = 0x64086408u;  // 1024 + 8 in each half
  static constexpr uint32_t kBase = 0x64006400u;   // 1024 in each half
  __device__ __forceinline__ static uint32_t zero_bias(uint32_t z) { return (0x6400u + z) * 0x00010001u; }
  __device__ __forceinline__ static uint32_t sub(uint32_t a, uint32_t b = 0x64086408u) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
  }
  __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
};

// Word w = 8 consecutive k (nibbles e0..e7 at bits 4i).  p[i] = (e_i, e_{i+4})
// as bf16x2 / f16x2: ((w >> 4i) & 0x000F000F) ^ magic, minus the bias.  For
// unsigned codes (the asymmetric scheme, ASYM) the XOR leaves the nibble as
// it is and `zb` = zero_bias(z) subtracts 128 + z (1024 + z), so p holds
// q - z exactly.
template <typename TX, bool ASYM = false>
__device__ __forceinline__ void expand(uint32_t w, uint32_t (&p)[4], uint32_t zb = Cvt<TX>::kMagic) {
  constexpr uint32_t kx = ASYM ? Cvt<TX>::kBase : Cvt<TX>::kMagic;
  const uint32_t v[4] = {w, w >> 4, w >> 8, w >> 12};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(v[i]), "r"(0x000F000Fu), "r"(kx));
    p[i] = Cvt<TX>::sub(r, ASYM ? zb : Cvt<TX>::kMagic);
  }
}

// x fragments for the pairing above: from x[k0 .. k0+8) = (x0x1, x2x3, x4x5,
// x6x7), MMA h = 0 takes (x0,x4), (x1,x5) and h = 1 takes (x2,x6), (x3,x7).
__device__ __forceinline__ uint4 pair_x(uint4 n) {
  return make_uint4(__byte_perm(n.x, n.z, 0x5410), __byte_perm(n.x, n.z, 0x7632),
                    __byte_perm(n.y, n.w, 0x5410), __byte_perm(n.y, n.w, 0x7632));
}

// The 8-k word (0..15 of a 128-k block) that lane c of a quad uses as its
// word j, for GPB groups per block (1: group multiple of 128, 2: group 64,
// 4: group 32); all four lanes of a quad then read the same group for word j.
template <int GPB>
__device__ __forceinline__ int word_index(int c, int j) {
  if (GPB == 1) return 4 * c + j;
  if (GPB == 2) return (j >> 1) * 8 + 2 * c + (j & 1);
  return 4 * j + c;
}

// The W tile row that MMA row g (0..7, and g + 8) of a 16-row tile reads.
// Rows are permuted inside the tile so that the lanes served by one shared-
// memory wavefront hit distinct 16-byte bank groups under the 128-byte
// swizzle (chunk c of row r sits at c ^ (r & 7)): 8 lanes per wavefront for
// the 16-byte loads (group multiple of 128), 16 for the 8-byte loads (group
// 64); 4-byte loads (group 32) are conflict-free in row order.
template <int GPB>
__device__ __forceinline__ int tile_row(int g) {
  if (GPB == 1) return (g >> 1) | ((g & 1) << 2);
  if (GPB == 2) return ((g & 3) << 1) | (g >> 2);
  return g;
}

struct WaitCtx {
  volatile uint32_t* abort;
  uint32_t* status;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const WaitCtx& w) {
#if INT4_DECODE_WAIT_MODE == 1
  if (ptx::mbar_test_wait(bar, parity)) return true;
#else
  if (ptx::mbar_try_wait(bar, parity)) return true;
#endif
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t i = 1; i != 0; ++i) {
#if INT4_DECODE_WAIT_MODE == 1
    if (ptx::mbar_test_wait(bar, parity)) return true;
#elif INT4_DECODE_WAIT_MODE == 2
    if (ptx::mbar_try_wait_sleep(bar, parity, 500u)) return true;
#else
    if (ptx::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
#endif
    if ((i & 15u) == 0u) {
      if (*w.abort) return false;
      if (ptx::globaltimer() - t0 > kTimeoutNs) break;
    }
  }
  *w.abort = 1u;
  report_status(w.status, kStatusTimeout);
  return false;
}

__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  for (uint32_t i = 0; i != 0xFFFFFFFFu; ++i) {
    if (ptx::mbar_try_wait(bar, parity)) return;
    if ((i & 127u) == 0u && ptx::globaltimer() - t0 > kTimeoutNs) return;
  }
}

template <int NT>
struct DLayout {
  static constexpr int kTiles = Tiles<NT>::kTiles;
  static constexpr int kWBytes = Tiles<NT>::kWBytes;
  // Per stage: W tile (1024-aligned for the swizzle), then the x tile with
  // room for NT * 8 rows (the copies write rows 0..M-1).
  static constexpr int kXSub = NT * 8 * 256 * 2;          // x rows of one sub-tile
  static constexpr int kXBytes = kSub * kXSub;
  static constexpr int kStageBytes = kWBytes + kXBytes;   // multiple of 1024
  static constexpr int offRed = kStages * kStageBytes;
  static constexpr int kRedBytes = kConsumers * kTiles * NT * 4 * 32 * 4;
  static constexpr int offBar = offRed + kRedBytes;
  static constexpr int offMisc = offBar + 2 * kStages * 8;
  static constexpr int kBytes = offMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <typename TX, int NT, int GPB, bool ASYM>
__global__ void __launch_bounds__(kThreads, INT4_DECODE_MIN_BLOCKS) decode_kernel(
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros, Epilogue ep,
    float* __restrict__ y, int64_t K, int group, int G, int M,
    int64_t N, int KB, int64_t U, int P, int64_t gran, float* __restrict__ partials,
    uint32_t* __restrict__ counters, uint32_t* status) {
  using L = DLayout<NT>;
  constexpr int kTiles = Tiles<NT>::kTiles;
  constexpr int kRowsPerCta = Tiles<NT>::kRowsPerCta;
  constexpr int kWBytes = Tiles<NT>::kWBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* empty = full + kStages;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::offMisc);
  volatile uint32_t* last_flag = abort_flag + 1;
  float* red = reinterpret_cast<float*>(smem + L::offRed);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Stream-K split: the units are (row tile, 128-k block) pairs in row-major
  // order, and CTA p takes units [p U / P, (p + 1) U / P).  Only the first
  // and the last segment of a run can be a partial tile; a tile the run
  // covers whole goes straight to y, a partial tile to its partial slot (2p
  // for the run's first segment when that starts inside a tile, else 2p + 1),
  // summed by the tile's last contributor to finish.
  // Runs start and end on multiples of `gran` units: 1 (any block, the
  // split) or KB (whole tiles, no partial tile: the schedule without scratch).
  const int64_t runs = U / gran;
  const int64_t u_begin = static_cast<int64_t>(blockIdx.x) * runs / P * gran;
  const int64_t u_end = static_cast<int64_t>(blockIdx.x + 1) * runs / P * gran;
  const uint32_t xbytes = static_cast<uint32_t>(M) * kSK * 128 * 2;  // all sub-tiles
  const WaitCtx wc{abort_flag, status};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[s]), kConsumers);
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_w);
    ptx::prefetch_tmap(&tm_x);
  }
  __syncthreads();
  // Launched as a programmatic dependent of what precedes it on the stream:
  // the set-up above overlaps that kernel's tail; every thread waits for it
  // to complete before reading an input or writing an output.
  ptx::launch_dependents();
  ptx::grid_dependency_wait();

  const int c = lane & 3;
  const int g = lane >> 2;
  const int cw = warp - 1;          // consumer index
  const int rg = cw % kRowGroups;   // row group of this consumer
  const int bs = cw / kRowGroups;   // which K block of each stage it takes

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int gs = 0;  // stages issued so far (ring slot and phase)
      bool ok = true;
      for (int64_t u = u_begin; ok && u < u_end;) {
        const int64_t r = u / KB;
        const int blo = static_cast<int>(u - r * KB);
        const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
        const int32_t row0 = static_cast<int32_t>(r * kRowsPerCta);
        for (int kb = blo; kb < bhi; kb += kSK, ++gs) {
          const int s = gs % kStages;
          if (!wait_bar(ptx::smem_u32(&empty[s]), ((gs / kStages) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * L::kStageBytes;
          ptx::mbar_arrive_expect_tx(ptx::smem_u32(&full[s]), kWBytes + xbytes);
#pragma unroll
          for (int q = 0; q < kSub; ++q) {
            ptx::tma_load_2d(st + q * (kWBytes / kSub), &tm_w, (kb + 2 * q) * 64, row0,
                             ptx::smem_u32(&full[s]));
            ptx::tma_load_2d(st + kWBytes + q * L::kXSub, &tm_x, (kb + 2 * q) * 128, 0,
                             ptx::smem_u32(&full[s]));
          }
        }
        u = r * KB + bhi;
      }
      if (*abort_flag) {
        // Wait (bounded) for the copies that may still be in flight.
        const int first = gs - kStages > 0 ? gs - kStages : 0;
        for (int j = first; j < gs; ++j) drain_bar(ptx::smem_u32(&full[j % kStages]), (j / kStages) & 1);
      }
    }
  } else {
    // ---------------- consumers ----------------
    // Each consumer owns kTiles 16-row tiles of row group rg and K block `bs`
    // of every stage.  Offsets within a stage are fixed per lane.
    constexpr int kW = (GPB == 1) ? 1 : (GPB == 2 ? 2 : 4);  // shared loads per row
    const int bl = bs & 1;                                   // block within its 256-k sub-tile
    const uint32_t sub_w = static_cast<uint32_t>((bs >> 1) * (kWBytes / kSub));
    uint32_t wofs[kTiles][2][kW];
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = rg * 16 * kTiles + 16 * t + tile_row<GPB>(g) + 8 * h;  // row within the W tile
        const int sw = r & 7;
#pragma unroll
        for (int q = 0; q < kW; ++q) {
          const int off = (GPB == 1) ? bl * 64 + 16 * c
                                     : (GPB == 2 ? bl * 64 + 32 * q + 8 * c : bl * 64 + 16 * q + 4 * c);
          wofs[t][h][q] = sub_w + static_cast<uint32_t>(r * 128 + ((((off >> 4) ^ sw)) << 4) + (off & 15));
        }
      }
    uint32_t xofs[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      xofs[j] = static_cast<uint32_t>(kWBytes + (bs >> 1) * L::kXSub +
                                      (g * 256 + bl * 128 + 8 * word_index<GPB>(c, j)) * 2);
    const int bpg = group / 128;  // K blocks per group when GPB == 1
    constexpr int kPer = kRowGroups * kTiles * NT * 4 * 32;  // outputs of a tile
    int gs = 0;
    for (int64_t u = u_begin; u < u_end;) {
      const int64_t r = u / KB;
      const int blo = static_cast<int>(u - r * KB);
      const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
      const int64_t row0 = r * kRowsPerCta;
      const uint16_t* sp[kTiles][2];
      const uint8_t* zp[kTiles][2];
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int64_t gr = row0 + rg * 16 * kTiles + 16 * t + tile_row<GPB>(g) + 8 * h;
          if (gr >= N) gr = N - 1;  // never written; keeps the scale load in bounds
          sp[t][h] = scales + gr * G;
          zp[t][h] = ASYM ? zeros + gr * G : nullptr;
        }
      float tot[kTiles][NT][4];
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) tot[t][nt][i] = 0.0f;
      bool ok = true;
      for (int kb_stage = blo; kb_stage < bhi; kb_stage += kSK, ++gs) {
        const int s = gs % kStages;
        // Every lane polls the barrier (its completion makes the copied bytes
        // visible to the lane); the vote keeps the warp together if a bounded
        // wait gave up in some lanes only.
        ok = __all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&full[s]), (gs / kStages) & 1, wc));
        if (!ok) break;
        const uint32_t st = sbase + s * L::kStageBytes;
        const int kb = kb_stage + bs;
        if (kb < bhi) {
        // This lane's four 8-k words of each of its rows.
        uint32_t wv[kTiles][2][4];
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (GPB == 1) {
              const uint4 u = ptx::lds128(st + wofs[t][h][0]);
              wv[t][h][0] = u.x; wv[t][h][1] = u.y; wv[t][h][2] = u.z; wv[t][h][3] = u.w;
            } else if (GPB == 2) {
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const uint2 u = ptx::lds64(st + wofs[t][h][q]);
                wv[t][h][2 * q] = u.x; wv[t][h][2 * q + 1] = u.y;
              }
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) wv[t][h][q] = ptx::lds32(st + wofs[t][h][q]);
            }
          }
        // All x fragments of this block.  Lanes of padding batch rows (n >= M)
        // take zeros without touching shared memory, which at small M saves
        // most of the x wavefronts (the rows share bank groups).
        uint4 xf4[4][NT];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            xf4[j][nt] = (g + 8 * nt < M) ? ptx::lds128(st + xofs[j] + nt * 8 * 512) : make_uint4(0u, 0u, 0u, 0u);
        // The block's scales (one per row and group) are loaded before they
        // are needed, as raw fp16 bits (two per register for group 64); group
        // 32 loads them at use, to stay within registers.
        uint32_t sraw[kTiles][2];
        uint32_t zraw[kTiles][2];  // zero points of the block's groups, one byte each
        if (GPB <= 2) {
          const int gi0 = (GPB == 1) ? ((bpg == 1) ? kb : kb / bpg) : kb * 2;
#pragma unroll
          for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t r = (gi0 < G) ? __ldg(sp[t][h] + gi0) : 0u;
              if (GPB == 2) r |= (gi0 + 1 < G) ? static_cast<uint32_t>(__ldg(sp[t][h] + gi0 + 1)) << 16 : 0u;
              sraw[t][h] = r;
            }
        }
        if (ASYM) {
#pragma unroll
          for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t r = 0u;
#pragma unroll
              for (int a = 0; a < GPB; ++a) {
                const int gi = (GPB == 1) ? ((bpg == 1) ? kb : kb / bpg) : kb * GPB + a;
                r |= (gi < G) ? static_cast<uint32_t>(__ldg(zp[t][h] + gi)) << (8 * a) : 0u;
              }
              zraw[t][h] = r;
            }
        }
        float acc[kTiles][NT][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // The accumulator restarts at the first word of each group.
          const bool first = (GPB == 1) ? (j == 0) : (GPB == 2 ? (j % 2 == 0) : true);
          const bool last = (GPB == 1) ? (j == 3) : (GPB == 2 ? (j % 2 == 1) : true);
          if (first) {
#pragma unroll
            for (int t = 0; t < kTiles; ++t)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[t][nt][i] = 0.0f;
          }
          uint4 xf[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) xf[nt] = pair_x(xf4[j][nt]);
#pragma unroll
          for (int t = 0; t < kTiles; ++t) {
            uint32_t pa[4], pb[4];
            if (ASYM) {
              const int a = (GPB == 1) ? 0 : (GPB == 2 ? (j >> 1) : j);  // the word's group in the block
              expand<TX, true>(wv[t][0][j], pa, Cvt<TX>::zero_bias((zraw[t][0] >> (8 * a)) & 0xFFu));
              expand<TX, true>(wv[t][1][j], pb, Cvt<TX>::zero_bias((zraw[t][1] >> (8 * a)) & 0xFFu));
            } else {
              expand<TX>(wv[t][0][j], pa);
              expand<TX>(wv[t][1][j], pb);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              Cvt<TX>::mma(acc[t][nt], pa[0], pb[0], pa[1], pb[1], xf[nt].x, xf[nt].y);
              Cvt<TX>::mma(acc[t][nt], pa[2], pb[2], pa[3], pb[3], xf[nt].z, xf[nt].w);
            }
          }
          if (last) {
            const int a = (GPB == 1) ? 0 : (GPB == 2 ? (j >> 1) : j);
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
              float sa, sb;
              if (GPB <= 2) {
                sa = f16_bits_to_float((sraw[t][0] >> (16 * a)) & 0xFFFFu);
                sb = f16_bits_to_float((sraw[t][1] >> (16 * a)) & 0xFFFFu);
              } else {
                const int gi = kb * GPB + a;
                const bool gok = gi < G;
                const int gc = gok ? gi : 0;
                sa = gok ? f16_bits_to_float(__ldg(sp[t][0] + gc)) : 0.0f;
                sb = gok ? f16_bits_to_float(__ldg(sp[t][1] + gc)) : 0.0f;
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                tot[t][nt][0] = fmaf(acc[t][nt][0], sa, tot[t][nt][0]);
                tot[t][nt][1] = fmaf(acc[t][nt][1], sa, tot[t][nt][1]);
                tot[t][nt][2] = fmaf(acc[t][nt][2], sb, tot[t][nt][2]);
                tot[t][nt][3] = fmaf(acc[t][nt][3], sb, tot[t][nt][3]);
              }
            }
          }
        }
      }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&empty[s]));
      }
      // Segment end: the two K-block slots of each row group are summed in a
      // fixed order.  The first barrier also agrees on whether any wait gave
      // up, so that every consumer leaves the loop at the same segment.
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            red[(((cw * kTiles + t) * NT + nt) * 4 + i) * 32 + lane] = tot[t][nt][i];
      const bool stop = ptx::bar_red_or(1, kConsumers * 32, !ok || *abort_flag != 0u);
      const bool whole = (blo == 0 && bhi == KB);
      if (!stop) {
        float* dst = whole ? nullptr
                           : partials + (2 * static_cast<int64_t>(blockIdx.x) + (blo == 0 ? 1 : 0)) * kPer;
        for (int e = threadIdx.x - 32; e < kPer; e += kConsumers * 32) {
          float sum = 0.0f;
#pragma unroll
          for (int q = 0; q < kSK; ++q) sum += red[q * kPer + e];
          if (!whole) {
            dst[e] = sum;
            continue;
          }
          const int ln = e & 31;
          const int i = (e >> 5) & 3;
          const int nt = (e >> 7) % NT;
          const int tw = (e >> 7) / NT;  // rg * kTiles + t
          const int m = nt * 8 + 2 * (ln & 3) + (i & 1);
          const int64_t row = row0 + tw * 16 + tile_row<GPB>(ln >> 2) + ((i < 2) ? 0 : 8);
          if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
        }
      }
      ptx::bar_sync(1, kConsumers * 32);  // red is rewritten by the next segment
      if (stop) break;
      if (!whole) {
        // Tile r straddles runs.  Its contributors are CTAs p_first..p_last
        // (p_first: the last run starting at or before the tile start); each
        // counts its arrival, and the last to arrive adds the pieces in CTA
        // order (p_first's is its run's last segment, slot 2p + 1; every later
        // one starts inside the tile, slot 2p), writes y and resets the count.
        const int64_t t0 = r * KB, t1 = (r + 1) * KB;
        const int p_first = static_cast<int>(((t0 + 1) * P + U - 1) / U - 1);
        const int p_last = static_cast<int>((t1 * P + U - 1) / U - 1);
        if (cw == 0 && lane == 0) {
          // The barrier above orders the CTA's partial stores before this
          // fence; fence and count release them to the last contributor.
          __threadfence();
          const uint32_t before = atomicAdd(&counters[p_first], 1u);
          const bool last = before == static_cast<uint32_t>(p_last - p_first);
          if (last) __threadfence();
          *last_flag = last ? 1u : 0u;
        }
        ptx::bar_sync(1, kConsumers * 32);
        if (*last_flag) {
          const float* first = partials + (2 * static_cast<int64_t>(p_first) + 1) * kPer;
          const float* rest = partials + 2 * static_cast<int64_t>(p_first + 1) * kPer;
          const int n_rest = p_last - p_first;
          for (int e = threadIdx.x - 32; e < kPer; e += kConsumers * 32) {
            float sum = __ldcg(first + e);
            for (int q = 0; q < n_rest; ++q) sum += __ldcg(rest + static_cast<int64_t>(2 * q) * kPer + e);
            const int ln = e & 31;
            const int i = (e >> 5) & 3;
            const int nt = (e >> 7) % NT;
            const int tw = (e >> 7) / NT;
            const int m = nt * 8 + 2 * (ln & 3) + (i & 1);
            const int64_t row = row0 + tw * 16 + tile_row<GPB>(ln >> 2) + ((i < 2) ? 0 : 8);
            if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
          }
          if (cw == 0 && lane == 0) counters[p_first] = 0u;
        }
      }
      u = r * KB + bhi;
    }
  }
}

// ---------------- integer-MMA decode (group a multiple of 128) ----------------
// The weights enter the int8 warp MMA as they are stored: the high nibble of
// a byte, masked in place, is the int8 value 16 q, and the low nibble is the
// same after a 4-bit left shift; two logic operations and a shift per 8
// weights, against eleven for the bf16 expansion.  x is split once per call
// (x_digits_kernel) into base-256 digits: for batch row m and 128-k block b,
// with e the binary exponent of the block's largest |x| (2^e <= max < 2^(e+1)),
//   v = rint(x 2^(29-e)),  |v| < 2^30,  v = d0 + 2^8 d1 + 2^16 d2 + 2^24 d3,
// with signed digits d_i (d0..d2 in [-128, 127], d3 in [-64, 64]).  v is x
// exactly whenever x 2^(29-e) is an integer: for every bf16 x within 2^22 of
// the block's largest magnitude (fp16: 2^19), zeros, and smaller values whose
// low significand bits are zero.  The MMA sums S_i = sum_k (16 q) d_i over the
// block exactly in int32 (|S_i| <= 2^21), and the block's x.q is
//   sum_k x q = 2^(e-33) (P01 + 2^16 P23),  P01 = S0 + 2^8 S1,  P23 = S2 + 2^8 S3,
// both P below 2^30, so the block needs two int-to-float conversions per
// output; the group's scale multiplies the block sum before the fp32 running
// sum, as on the page.  The four digits of row m sit in four MMA columns, so
// one n = 8 MMA serves two batch rows: lane c of a quad holds columns 2c and
// 2c + 1, i.e. P01 (c even) or P23 (c odd) of row 2nt + c / 2, and the two
// halves are added when the tile is written (the odd lanes' 2^16 rides on the
// scale they multiply by, which is exact).
//
// A block row that some value does not fit exactly (a block spanning more
// than that range, values below 2^-93 times a power of two, NaN or infinity)
// is flagged in its record, and the consumers compute that block on the
// 16-bit MMA with x as stored instead (the bf16/fp16 products are exact, as in
// decode_kernel).  So the integer form never rounds x, and the result meets
// the accuracy of the floating-point path on every input.
//
// Digit record of one 128-k block: NP n-tiles of 1 KB (8 columns x 128 k, one
// byte each, in MMA fragment order), then 16 fp32 factors 2^(e-33) (one per
// batch row), then 16 flag bytes (non-zero: the row's block takes the 16-bit
// path), then padding to 128 bytes.  Column col of an n-tile holds digit
// col % 4 of row 2nt + col / 4; inside a column, the 16-byte chunk
// ((2c + j / 2) ^ (col & 1)) holds, at byte 8 (j % 2), the B fragment of lane c
// for the MMA over words 4c + j of the block's 16 words: 4 digits of the
// word's even k, then 4 of its odd k.  The XOR spreads the 16-byte loads of a
// quarter warp over all banks.
constexpr int kDigitTile = 1024;
constexpr int kRecFlags = 64;  // flag bytes of a record, after its factors
// Per batch row m (records of at most two n-tiles): the block's digit sums
// C01 = D0 + 256 D1 and C23 = D2 + 256 D3 (D_i = the sum of digit i over the
// block's k) as two int32 at kRecSums + 8 m; the affine scheme subtracts
// z C from each pair product.
constexpr int kRecSums = 96;

__device__ __forceinline__ void transpose4x4(uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                             uint32_t (&o)[4]) {
  const uint32_t ab_lo = __byte_perm(a, b, 0x5140);  // a0 b0 a1 b1
  const uint32_t ab_hi = __byte_perm(a, b, 0x7362);  // a2 b2 a3 b3
  const uint32_t cd_lo = __byte_perm(c, d, 0x5140);
  const uint32_t cd_hi = __byte_perm(c, d, 0x7362);
  o[0] = __byte_perm(ab_lo, cd_lo, 0x5410);  // a0 b0 c0 d0
  o[1] = __byte_perm(ab_lo, cd_lo, 0x7632);  // a1 b1 c1 d1
  o[2] = __byte_perm(ab_hi, cd_hi, 0x5410);  // a2 b2 c2 d2
  o[3] = __byte_perm(ab_hi, cd_hi, 0x7632);  // a3 b3 c3 d3
}

// 8 x values (one 8-k word) from 16 bytes of bf16 or fp16, exactly.
template <typename TX>
__device__ __forceinline__ void word_as_float(uint4 u, float (&v)[8]);
template <>
__device__ __forceinline__ void word_as_float<__nv_bfloat16>(uint4 u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void word_as_float<__half>(uint4 u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// Bits of the largest |x| of a 128-k block (8 values per lane, 16 lanes: a
// half warp), as an unsigned max over the magnitude bits, which orders every
// finite value below infinity and infinity below NaN.  All 32 lanes must call
// it together.
__device__ __forceinline__ uint32_t block_absmax_bits(const float (&v)[8]) {
  uint32_t mb = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) mb = max(mb, __float_as_uint(v[i]) & 0x7FFFFFFFu);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  return mb;
}

// The digits of one word of a block: ev[i] / od[i] hold digit i of the
// word's even / odd k (one byte each, k order), f the block's factor
// 2^(e-33), and `inexact` whether some value of the word is not an integer
// multiple of 2^(e-29) (or the block holds a NaN or an infinity): the block
// row is then flagged for the 16-bit path.  A block of zeros gives zero
// digits and factor.  Blocks whose largest |x| is below 2^-93 are scaled as if
// it were 2^-93, which keeps the factors normal floats.
__device__ __forceinline__ void word_digits(const float (&v)[8], uint32_t amax_bits,
                                            uint32_t (&ev)[4], uint32_t (&od)[4], float& f,
                                            bool& inexact) {
  uint32_t dd[8];
  f = 0.0f;
  inexact = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) dd[i] = 0u;
  if (amax_bits >= 0x7F800000u) {
    inexact = true;
  } else if (amax_bits != 0u) {
    // The exponent field (subnormals read as -127, below the clamp).
    int e = static_cast<int>(amax_bits >> 23) - 127;
    if (e < -93) e = -93;
    const int p = 29 - e;  // in [-98, 122]: two normal power-of-two factors
    const int p1 = p >> 1, p2 = p - p1;
    const float s1 = __uint_as_float(static_cast<uint32_t>(p1 + 127) << 23);
    const float s2 = __uint_as_float(static_cast<uint32_t>(p2 + 127) << 23);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // t = x 2^p: exact unless it underflows, which can only happen for p < 0
      // and leaves |t| < 2^-126, never a non-zero integer (hence the guard).
      const float t = (v[i] * s1) * s2;
      const int vi = __float2int_rn(t);
      // Balanced base-256 digits: the bytes of v + 0x808080 with the low three
      // flipped back by 128.
      dd[i] = (static_cast<uint32_t>(vi) + 0x808080u) ^ 0x808080u;
      inexact |= (rintf(t) != t) | ((t == 0.0f) & (v[i] != 0.0f));
    }
    f = __uint_as_float(static_cast<uint32_t>(e - 33 + 127) << 23);
  }
  transpose4x4(dd[0], dd[2], dd[4], dd[6], ev);
  transpose4x4(dd[1], dd[3], dd[5], dd[7], od);
}

// The block's digit-pair sums (C01, C23) from each lane's digit words ev/od
// (signed bytes), summed over the half warp.  All 32 lanes call it together.
__device__ __forceinline__ int2 block_digit_sums(const uint32_t (&ev)[4], const uint32_t (&od)[4]) {
  int d[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = __dp4a(static_cast<int>(ev[i]), 0x01010101, __dp4a(static_cast<int>(od[i]), 0x01010101, 0));
  // The pair sums are linear in the digits: reduce them directly.
  int c01 = d[0] + 256 * d[1], c23 = d[2] + 256 * d[3];
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    c01 += __shfl_xor_sync(0xffffffffu, c01, o);
    c23 += __shfl_xor_sync(0xffffffffu, c23, o);
  }
  return make_int2(c01, c23);
}

// Whether any lane of this lane's half warp (one block) set `pred`.  All 32
// lanes must call it together.
__device__ __forceinline__ bool half_warp_any(bool pred) {
  const uint32_t bal = __ballot_sync(0xffffffffu, pred);
  return ((bal >> (threadIdx.x & 16u)) & 0xFFFFu) != 0u;
}

// Byte offset, inside a record, of the fragment pair (digit i of row m, word h).
__device__ __forceinline__ int digit_offset(int m, int i, int h) {
  const int col = 4 * (m & 1) + i;
  const int c = h >> 2, j = h & 3;
  return (m >> 1) * kDigitTile + col * 128 + (((2 * c + (j >> 1)) ^ (col & 1)) << 4) + (j & 1) * 8;
}

// Digit records of rows 0 .. R-1 of one block from its x rows in shared
// memory (row pitch 512 bytes): xs addresses this lane's word h of row 0, rb
// the block's record.  All 32 lanes call it together (one block per half
// warp).
template <typename TX, int R, int NP, bool SUMS>
__device__ __forceinline__ void convert_rows(uint32_t xs, uint32_t rb, int h) {
  static_assert(R <= 4, "the flag bytes of the converted rows share one word");
  float v[R][8];
  uint32_t mb[R];
#pragma unroll
  for (int r = 0; r < R; ++r) word_as_float<TX>(ptx::lds128(xs + r * 512), v[r]);
#pragma unroll
  for (int r = 0; r < R; ++r) mb[r] = block_absmax_bits(v[r]);
  uint32_t flags = 0u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    uint32_t ev[4], od[4];
    float f;
    bool inexact;
    word_digits(v[r], mb[r], ev, od, f, inexact);
    if (half_warp_any(inexact)) flags |= 1u << (8 * r);
#pragma unroll
    for (int i = 0; i < 4; ++i) ptx::sts64(rb + digit_offset(r, i, h), ev[i], od[i]);
    if (h == 0) ptx::sts32(rb + NP * kDigitTile + 4 * r, __float_as_uint(f));
    if (SUMS) {
      const int2 cs = block_digit_sums(ev, od);
      if (h == 0) ptx::sts64(rb + NP * kDigitTile + kRecSums + 8 * r, static_cast<uint32_t>(cs.x), static_cast<uint32_t>(cs.y));
    }
  }
  // Rows R .. 3 of the word stay zero (rows past M are never written).
  if (h == 0) ptx::sts32(rb + NP * kDigitTile + kRecFlags, flags);
}

// One half warp per (batch row m < MP, record b < nrec); lane h takes the
// 8-k word h of the block.  Rows m >= M and k >= K are zero.
template <typename TX>
__global__ void __launch_bounds__(256) x_digits_kernel(const TX* __restrict__ x, int64_t K, int M,
                                                      int MP, int NP, int64_t nrec,
                                                      uint8_t* __restrict__ rec) {
  // Launched as a programmatic dependent: the matmul grid may start its
  // set-up now; this grid waits for the kernel before it (which may write x,
  // or still read the records) to complete.
  ptx::launch_dependents();
  ptx::grid_dependency_wait();
  const int64_t hw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int h = threadIdx.x & 15;
  const bool live = hw < static_cast<int64_t>(MP) * nrec;
  const int m = live ? static_cast<int>(hw % MP) : 0;
  const int64_t b = live ? hw / MP : 0;
  const int64_t k0 = b * 128 + 8 * h;
  float v[8];
  if (live && m < M && k0 < K) {
    word_as_float<TX>(__ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k0)), v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
  const uint32_t amax_bits = block_absmax_bits(v);
  uint32_t ev[4], od[4];
  float f;
  bool inexact;
  word_digits(v, amax_bits, ev, od, f, inexact);
  const bool flag = half_warp_any(inexact);  // every lane votes, live or not
  const int2 cs = block_digit_sums(ev, od);   // every lane takes part
  if (!live) return;
  uint8_t* r = rec + b * (static_cast<int64_t>(NP) * kDigitTile + 128);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint2*>(r + digit_offset(m, i, h)) = make_uint2(ev[i], od[i]);
  if (h == 0) {
    reinterpret_cast<float*>(r + NP * kDigitTile)[m] = f;
    r[NP * kDigitTile + kRecFlags + m] = flag ? 1u : 0u;
    if (NP <= 2) *reinterpret_cast<int2*>(r + NP * kDigitTile + kRecSums + 8 * m) = cs;
  }
}

// Shape of the integer-MMA decode for NP n-tiles (batch rows up to 2 NP).
// FUSE (M <= 2): the kernel converts x itself; a converter warp turns each
// stage's x tile (copied on its own barrier, ahead of the weights) into the
// stage's digit records, so one launch does the whole call.  For larger M
// that per-CTA conversion would cost more than the matmul, and
// x_digits_kernel writes the records once per call.
template <int NP, bool FUSE>
struct I8Shape {
  static constexpr bool kFuse = FUSE;                                // converter warp in the CTA
  static_assert(!FUSE || NP == 1, "the converter warp serves up to two batch rows");
  static constexpr int kTiles = NP <= 2 ? INT4_DECODE_I8_TILES : 1;  // 16-row tiles per consumer
  static constexpr int kRowsPerCta = 16 * kTiles * kRowGroups;       // 128 or 64
  static constexpr int kWBytes = kRowsPerCta * kSK * 64;             // packed W of a stage
  static constexpr int kRec = NP * kDigitTile + 128;                 // digit record of a block
  static constexpr int kXBytes = kFuse ? 2 * NP * 256 * 2 : 0;       // x rows of the stage (fused)
  static constexpr int offX = kWBytes + kSK * kRec;                  // within a stage
  static constexpr int kStageBytes = (offX + kXBytes + 1023) / 1024 * 1024;
  static constexpr int kRedPer = kRowGroups * kTiles * NP * 2 * 32;  // lane sums of one K slot
  static constexpr int kOut = kRowGroups * kTiles * NP * 2 * 16;     // (row, batch row) outputs of a tile
  static constexpr int kThreads = 32 * (kConsumers + 1 + (kFuse ? 1 : 0));
  static constexpr int offRed = kStages * kStageBytes;
  static constexpr int offBar = offRed + kSK * kRedPer * 4;
  static constexpr int offMisc = offBar + 4 * kStages * 8;
  static constexpr int kAlloc = offMisc + 16 + 1024;
  static constexpr int kMinBlocks = NP == 1 ? INT4_DECODE_I8_MINB1 : 2;  // CTAs per SM
  static_assert(kSK == 2, "a stage is one 256-k copy of W: K slot bs reads its 64-byte half");
  static_assert(offX % 128 == 0, "x tile copies need 128-byte aligned destinations");
};

__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Whether any of the 2 NP batch rows of a record is flagged (its flag bytes
// start at `a`, 16-byte aligned; bytes of rows past 2 NP are not read).
template <int NP>
__device__ __forceinline__ bool record_flagged(uint32_t a) {
  if (NP == 1) return (ptx::lds32(a) & 0xFFFFu) != 0u;
  if (NP == 2) return ptx::lds32(a) != 0u;
  if (NP == 4) {
    const uint2 f = ptx::lds64(a);
    return (f.x | f.y) != 0u;
  }
  const uint4 f = ptx::lds128(a);
  return (f.x | f.y | f.z | f.w) != 0u;
}

// Bytes q - z (int8, in [-15, 15]) of the four unsigned codes held one per
// byte in `q` (each 0..15), for zero point z (zz = z in every byte): with
// q | 0x80 the per-byte subtraction cannot borrow (128 + q - z >= 113), and
// flipping bit 7 back leaves the two's-complement q - z.
__device__ __forceinline__ uint32_t affine_bytes(uint32_t q, uint32_t zz) {
  return ((q | 0x80808080u) - zz) ^ 0x80808080u;
}

// One 128-k block (kb) of a flagged record, on the 16-bit warp MMA with x as
// stored, read from global memory (L2 holds it): the nibbles are expanded to
// bf16/fp16 and paired with x as in decode_kernel, so every product is exact
// and the block sums in fp32.  The MMA's columns are batch rows here (8 per
// n-tile), so each lane then fetches, for n-tile nt of the integer layout,
// the sums of its batch row 2nt + c / 2 from lane (g, nt % 4) of the quad
// row, and the even lanes add them (times the scale) to their totals.  wr
// holds words 4c .. 4c + 3 of rows g and g + 8 of each tile.  All 32 lanes
// call it together.
template <typename TX, int NP, int kTiles, bool ASYM>
__device__ __forceinline__ void block_fallback(const TX* __restrict__ x, int64_t K, int M, int kb,
                                               int g, int c, const uint4 (&wr)[kTiles][2],
                                               const float (&sa)[kTiles], const float (&sb)[kTiles],
                                               const uint32_t (&za)[kTiles], const uint32_t (&zb)[kTiles],
                                               float (&tot)[kTiles][NP][2]) {
  constexpr int NTB = (2 * NP + 7) / 8;  // 16-bit MMA n-tiles (8 batch rows each)
  float acc[kTiles][NTB][4];
#pragma unroll
  for (int t = 0; t < kTiles; ++t)
#pragma unroll
    for (int nb = 0; nb < NTB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][nb][i] = 0.0f;
  const int64_t k0 = static_cast<int64_t>(kb) * 128 + 32 * c;  // this lane's 32 k (K % 32 == 0)
  const bool kin = k0 < K;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 xf[NTB];
#pragma unroll
    for (int nb = 0; nb < NTB; ++nb) {
      const int m = 8 * nb + g;
      xf[nb] = (kin && m < M)
                   ? pair_x(__ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k0 + 8 * j)))
                   : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
      const uint32_t w0[4] = {wr[t][0].x, wr[t][0].y, wr[t][0].z, wr[t][0].w};
      const uint32_t w1[4] = {wr[t][1].x, wr[t][1].y, wr[t][1].z, wr[t][1].w};
      uint32_t pa[4], pb[4];
      expand<TX, ASYM>(w0[j], pa, ASYM ? Cvt<TX>::zero_bias(za[t]) : Cvt<TX>::kMagic);
      expand<TX, ASYM>(w1[j], pb, ASYM ? Cvt<TX>::zero_bias(zb[t]) : Cvt<TX>::kMagic);
#pragma unroll
      for (int nb = 0; nb < NTB; ++nb) {
        Cvt<TX>::mma(acc[t][nb], pa[0], pb[0], pa[1], pb[1], xf[nb].x, xf[nb].y);
        Cvt<TX>::mma(acc[t][nb], pa[2], pb[2], pa[3], pb[3], xf[nb].z, xf[nb].w);
      }
    }
  }
  const int lane_base = g << 2;
  const bool odd_row = (c >> 1) != 0;  // batch row 2nt + 1
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) {
    const int src = lane_base | (nt & 3);
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
      const float r0 = __shfl_sync(0xffffffffu, acc[t][nt >> 2][0], src);
      const float r1 = __shfl_sync(0xffffffffu, acc[t][nt >> 2][1], src);
      const float r2 = __shfl_sync(0xffffffffu, acc[t][nt >> 2][2], src);
      const float r3 = __shfl_sync(0xffffffffu, acc[t][nt >> 2][3], src);
      if ((c & 1) == 0) {
        tot[t][nt][0] = fmaf(odd_row ? r1 : r0, sa[t], tot[t][nt][0]);
        tot[t][nt][1] = fmaf(odd_row ? r3 : r2, sb[t], tot[t][nt][1]);
      }
    }
  }
}

// Same CTA roles, ring, stream-K split and last-contributor reduction as
// decode_kernel.  Each stage carries the digit records of its two blocks:
// converted in the CTA from the stage's x tile (FUSE), or one bulk copy of
// the records x_digits_kernel wrote.
template <typename TX, int NP, bool FUSE, bool ASYM>
__global__ void __launch_bounds__(I8Shape<NP, FUSE>::kThreads, I8Shape<NP, FUSE>::kMinBlocks) decode_i8_kernel(
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
    const TX* __restrict__ x, const uint8_t* __restrict__ rec,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros, Epilogue ep,
    float* __restrict__ y, int64_t K, int group, int G, int M,
    int64_t N, int KB, int64_t U, int P, int64_t gran, float* __restrict__ partials,
    uint32_t* __restrict__ counters, uint32_t* status) {
  using S = I8Shape<NP, FUSE>;
  // Affine codes as unsigned q with z times the block's digit sums
  // subtracted (records of at most two n-tiles carry the sums).
  constexpr bool kAsymSums = ASYM && NP <= 2;
  constexpr int kTiles = S::kTiles;
  constexpr int kRowsPerCta = S::kRowsPerCta;
  constexpr int kWBytes = S::kWBytes;
  constexpr int kRec = S::kRec;
  constexpr int kOut = S::kOut;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::offBar);
  uint64_t* empty = full + kStages;
  uint64_t* ready = empty + kStages;  // records of the stage written (fused)
  uint64_t* xfull = ready + kStages;  // x tile of the stage landed (fused)
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::offMisc);
  volatile uint32_t* last_flag = abort_flag + 1;
  float* red = reinterpret_cast<float*>(smem + S::offRed);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Runs start and end on multiples of `gran` units: 1 (any block, the
  // split) or KB (whole tiles, no partial tile: the schedule without scratch).
  const int64_t runs = U / gran;
  const int64_t u_begin = static_cast<int64_t>(blockIdx.x) * runs / P * gran;
  const int64_t u_end = static_cast<int64_t>(blockIdx.x + 1) * runs / P * gran;
  const WaitCtx wc{abort_flag, status};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&empty[s]), kConsumers);
      ptx::mbar_init(ptx::smem_u32(&ready[s]), 1);
      ptx::mbar_init(ptx::smem_u32(&xfull[s]), 1);
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_w);
    if (S::kFuse) ptx::prefetch_tmap(&tm_x);
  }
  __syncthreads();
  // Launched as a programmatic dependent of what precedes it on the stream
  // (the digits grid, or any kernel): the set-up above overlaps that grid's
  // tail, and every thread waits for it to complete (its writes visible)
  // before reading an input or writing an output.  Before that wait the
  // producer only asks L2 to prefetch the weight tiles of its first stages
  // (L2 is coherent, so a tile the earlier kernel still writes is read
  // fresh after the wait).  The next kernel may likewise start early.
  if (warp == 0 && lane == 0) {
    int pf = 0;
    for (int64_t u = u_begin; pf < kStages && u < u_end;) {
      const int64_t r = u / KB;
      const int blo = static_cast<int>(u - r * KB);
      const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
      for (int kb = blo; pf < kStages && kb < bhi; kb += kSK, ++pf)
        ptx::tma_prefetch_2d(&tm_w, kb * 64, static_cast<int32_t>(r * kRowsPerCta));
      u = r * KB + bhi;
    }
  }
  ptx::launch_dependents();
  ptx::grid_dependency_wait();

  const int c = lane & 3;
  const int g = lane >> 2;
  const int cw = warp - 1;
  const int rg = cw % kRowGroups;
  const int bs = cw / kRowGroups;

  if (S::kFuse && warp == kConsumers + 1) {
    // ---------------- converter (NP <= 2) ----------------
    // Rows M .. 2NP - 1 of every record stay zero: cleared once here, before
    // the first stage is declared ready.
    for (int o = lane * 16; o < kStages * S::kStageBytes; o += 32 * 16) {
      const int ws = o % S::kStageBytes;
      if (ws >= kWBytes && ws < S::offX) ptx::sts128(sbase + o, make_uint4(0u, 0u, 0u, 0u));
    }
    int nst = 0;  // stages of this CTA, counted as the producer issues them
    for (int64_t u = u_begin; u < u_end;) {
      const int64_t r = u / KB;
      const int blo = static_cast<int>(u - r * KB);
      const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
      nst += (bhi - blo + kSK - 1) / kSK;
      u = r * KB + bhi;
    }
    for (int gs = 0; gs < nst; ++gs) {
      const int s = gs % kStages;
      if (!__all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&xfull[s]), (gs / kStages) & 1, wc))) break;
      const uint32_t st = sbase + s * S::kStageBytes;
      // Half warp bl takes block bl of the stage, lane h its word h, for
      // every batch row (both rows' chains interleaved when M = 2).
      const int bl = lane >> 4, h = lane & 15;
      const uint32_t xs = st + S::offX + bl * 256 + 16 * h;
      const uint32_t rb = st + kWBytes + bl * kRec;
      if (M == 2)
        convert_rows<TX, 2, NP, kAsymSums>(xs, rb, h);
      else
        convert_rows<TX, 1, NP, kAsymSums>(xs, rb, h);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&ready[s]));
    }
  } else if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int gs = 0;
      bool ok = true;
      // A second cursor over the run, INT4_DECODE_L2_AHEAD stages beyond the
      // ring (the first kStages stages were prefetched before the dependency
      // wait): each issued stage asks L2 to prefetch the weights of that
      // later stage, more bytes in flight without more shared memory.
      constexpr int kAheadL2 = INT4_DECODE_L2_AHEAD;
      int64_t pu = u_begin, pr = u_begin / KB;
      int pkb = static_cast<int>(u_begin - pr * KB);
      int pbhi = static_cast<int>((u_end - pr * KB < KB) ? u_end - pr * KB : KB);
      auto pf_advance = [&]() {
        pkb += kSK;
        if (pkb >= pbhi) {
          pu = pr * KB + pbhi;
          pr = pu / KB;
          pkb = static_cast<int>(pu - pr * KB);
          pbhi = static_cast<int>((u_end - pr * KB < KB) ? u_end - pr * KB : KB);
        }
      };
      if (kAheadL2 > 0) {
        for (int j = 0; j < kStages && pu < u_end; ++j) pf_advance();   // prefetched at the start
        for (int j = 0; j < kAheadL2 - 1 && pu < u_end; ++j) {
          ptx::tma_prefetch_2d(&tm_w, pkb * 64, static_cast<int32_t>(pr * kRowsPerCta));
          pf_advance();
        }
      }
      for (int64_t u = u_begin; ok && u < u_end;) {
        const int64_t r = u / KB;
        const int blo = static_cast<int>(u - r * KB);
        const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
        const int32_t row0 = static_cast<int32_t>(r * kRowsPerCta);
        for (int kb = blo; kb < bhi; kb += kSK, ++gs) {
          const int s = gs % kStages;
          if (kAheadL2 > 0 && pu < u_end) {
            ptx::tma_prefetch_2d(&tm_w, pkb * 64, static_cast<int32_t>(pr * kRowsPerCta));
            pf_advance();
          }
          if (!wait_bar(ptx::smem_u32(&empty[s]), ((gs / kStages) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * S::kStageBytes;
          if (S::kFuse) {
            // The stage's x rows (256 k; past K the copy fills zeros) on their
            // own barrier, so the converter starts while W is in flight.
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(&xfull[s]), static_cast<uint32_t>(M) * 512);
            ptx::tma_load_2d(st + S::offX, &tm_x, kb * 128, 0, ptx::smem_u32(&xfull[s]));
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(&full[s]), kWBytes);
            ptx::tma_load_2d(st, &tm_w, kb * 64, row0, ptx::smem_u32(&full[s]));
            continue;
          }
          ptx::mbar_arrive_expect_tx(ptx::smem_u32(&full[s]), kWBytes + kSK * kRec);
          ptx::tma_load_2d(st, &tm_w, kb * 64, row0, ptx::smem_u32(&full[s]));
          ptx::bulk_load(st + kWBytes, rec + static_cast<int64_t>(kb) * kRec, kSK * kRec,
                         ptx::smem_u32(&full[s]));
        }
        u = r * KB + bhi;
      }
      if (*abort_flag) {
        const int first = gs - kStages > 0 ? gs - kStages : 0;
        for (int j = first; j < gs; ++j) {
          drain_bar(ptx::smem_u32(&full[j % kStages]), (j / kStages) & 1);
          if (S::kFuse) drain_bar(ptx::smem_u32(&xfull[j % kStages]), (j / kStages) & 1);
        }
      }
    }
  } else {
    // ---------------- consumers ----------------
    // Consumer (rg, bs) takes kTiles 16-row tiles of row group rg and K block
    // bs of every stage: per tile, lane (g, c) reads the 16 bytes (words
    // 4c .. 4c + 3) of rows g and g + 8 (permuted as in decode_kernel), one
    // word per MMA.
    uint32_t wofs[kTiles][2];
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = rg * 16 * kTiles + 16 * t + tile_row<1>(g) + 8 * h;
        const int off = bs * 64 + 16 * c;
        wofs[t][h] = static_cast<uint32_t>(r * 128 + (((off >> 4) ^ (r & 7)) << 4));
      }
    const uint32_t xrec = static_cast<uint32_t>(kWBytes + bs * kRec);
    uint32_t bofs[2];
#pragma unroll
    for (int jp = 0; jp < 2; ++jp)
      bofs[jp] = xrec + static_cast<uint32_t>(g * 128 + (((2 * c + jp) ^ (g & 1)) << 4));
    // Factor of batch row 2nt + c / 2 (plus 8 nt bytes); the odd lanes' P23
    // weighs 2^16 more, which they fold into their scale.
    const uint32_t fofs = xrec + static_cast<uint32_t>(NP * kDigitTile + 4 * (c >> 1));
    const uint32_t flagofs = xrec + static_cast<uint32_t>(NP * kDigitTile + kRecFlags);
    // This lane's digit-pair sum: batch row 2 nt + c / 2, pair c & 1 (plus 16 nt bytes).
    const uint32_t sumofs = xrec + static_cast<uint32_t>(NP * kDigitTile + kRecSums + 8 * (c >> 1) + 4 * (c & 1));
    // Affine codes enter the MMA as q (or q - z), not 16 q: 16 times the factor.
    const float lane_mul = ((c & 1) ? 65536.0f : 1.0f) * (ASYM ? 16.0f : 1.0f);
    const int bpg = group / 128;
    int gs = 0;
    for (int64_t u = u_begin; u < u_end;) {
      const int64_t r = u / KB;
      const int blo = static_cast<int>(u - r * KB);
      const int bhi = static_cast<int>((u_end - r * KB < KB) ? u_end - r * KB : KB);
      const int64_t row0 = r * kRowsPerCta;
      const uint16_t* sp[kTiles][2];
      const uint8_t* zp[kTiles][2];
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int64_t gr = row0 + rg * 16 * kTiles + 16 * t + tile_row<1>(g) + 8 * h;
          if (gr >= N) gr = N - 1;  // never written; keeps the scale load in bounds
          sp[t][h] = scales + gr * G;
          zp[t][h] = ASYM ? zeros + gr * G : nullptr;
        }
      float tot[kTiles][NP][2];
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NP; ++nt) tot[t][nt][0] = tot[t][nt][1] = 0.0f;
      // The scales of a block are loaded kAhead blocks ahead (a register
      // queue): a block's work is shorter than a load's latency.
      constexpr int kAhead = INT4_DECODE_I8_SCALE_AHEAD;
      uint16_t sraw[kAhead][kTiles][2];
      uint8_t zraw[kAhead][kTiles][2];
      auto load_scales = [&](int kb, uint16_t (&dst)[kTiles][2], uint8_t (&zdst)[kTiles][2]) {
        const int gi = (bpg == 1) ? kb : kb / bpg;
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          dst[t][0] = __ldg(sp[t][0] + gi);
          dst[t][1] = __ldg(sp[t][1] + gi);
          if (ASYM) {
            zdst[t][0] = __ldg(zp[t][0] + gi);
            zdst[t][1] = __ldg(zp[t][1] + gi);
          }
        }
      };
#pragma unroll
      for (int q = 0; q < kAhead; ++q)
        if (blo + bs + q * kSK < bhi) load_scales(blo + bs + q * kSK, sraw[q], zraw[q]);
      bool ok = true;
      for (int kb_stage = blo; kb_stage < bhi; kb_stage += kSK, ++gs) {
        const int s = gs % kStages;
        const int kb = kb_stage + bs;
        float sa[kTiles], sb[kTiles];
        uint32_t za[kTiles], zb[kTiles];
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          sa[t] = f16_bits_to_float(sraw[0][t][0]);
          sb[t] = f16_bits_to_float(sraw[0][t][1]);
          za[t] = ASYM ? zraw[0][t][0] : 0u;
          zb[t] = ASYM ? zraw[0][t][1] : 0u;
        }
#pragma unroll
        for (int q = 0; q + 1 < kAhead; ++q)
#pragma unroll
          for (int t = 0; t < kTiles; ++t) {
            sraw[q][t][0] = sraw[q + 1][t][0];
            sraw[q][t][1] = sraw[q + 1][t][1];
            zraw[q][t][0] = zraw[q + 1][t][0];
            zraw[q][t][1] = zraw[q + 1][t][1];
          }
        if (kb + kAhead * kSK < bhi) load_scales(kb + kAhead * kSK, sraw[kAhead - 1], zraw[kAhead - 1]);
        ok = __all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&full[s]), (gs / kStages) & 1, wc));
        if (ok && S::kFuse)
          ok = __all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&ready[s]), (gs / kStages) & 1, wc));
        if (!ok) break;
        const uint32_t st = sbase + s * S::kStageBytes;
        if (kb < bhi) {
          // The words of rows g and g + 8 of each tile (words 4c .. 4c + 3).
          uint4 wr[kTiles][2];
#pragma unroll
          for (int t = 0; t < kTiles; ++t) {
            wr[t][0] = ptx::lds128(st + wofs[t][0]);
            wr[t][1] = ptx::lds128(st + wofs[t][1]);
          }
          // At NP == 1 the block's digit fragments and factors are loaded
          // with the weights and the flags, before the test that branches on
          // the flags, so that all of these loads are in flight together.
          constexpr bool kHoist = NP == 1;
          constexpr int NPH = kHoist ? NP : 1;
          uint4 hb01[NPH], hb23[NPH];
          float hfct[NPH];
          if (kHoist) {
#pragma unroll
            for (int nt = 0; nt < NPH; ++nt) {
              hb01[nt] = ptx::lds128(st + bofs[0] + nt * kDigitTile);
              hb23[nt] = ptx::lds128(st + bofs[1] + nt * kDigitTile);
              hfct[nt] = __uint_as_float(ptx::lds32(st + fofs + nt * 8));
            }
          }
          if (__builtin_expect(record_flagged<NP>(st + flagofs), 0)) {
            // Some batch row's x does not fit its digits exactly: the whole
            // block runs on the 16-bit MMA with x as stored.
            block_fallback<TX, NP, kTiles, ASYM>(x, K, M, kb, g, c, wr, sa, sb, za, zb, tot);
          } else {
            // A fragments of the block's four MMAs (k32 each): rows g and
            // g + 8, low nibbles (shifted) in k slots 0..15, high nibbles in
            // 16..31.
            uint32_t a[kTiles][4][4];
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
              const uint32_t w0[4] = {wr[t][0].x, wr[t][0].y, wr[t][0].z, wr[t][0].w};
              const uint32_t w1[4] = {wr[t][1].x, wr[t][1].y, wr[t][1].z, wr[t][1].w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (kAsymSums) {
                  // The unsigned codes q; z times the block's digit sums is
                  // subtracted from the products below.
                  a[t][j][0] = w0[j] & 0x0F0F0F0Fu;
                  a[t][j][1] = w1[j] & 0x0F0F0F0Fu;
                  a[t][j][2] = (w0[j] >> 4) & 0x0F0F0F0Fu;
                  a[t][j][3] = (w1[j] >> 4) & 0x0F0F0F0Fu;
                } else if (ASYM) {
                  const uint32_t zza = za[t] * 0x01010101u, zzb = zb[t] * 0x01010101u;
                  a[t][j][0] = affine_bytes(w0[j] & 0x0F0F0F0Fu, zza);
                  a[t][j][1] = affine_bytes(w1[j] & 0x0F0F0F0Fu, zzb);
                  a[t][j][2] = affine_bytes((w0[j] >> 4) & 0x0F0F0F0Fu, zza);
                  a[t][j][3] = affine_bytes((w1[j] >> 4) & 0x0F0F0F0Fu, zzb);
                } else {
                  a[t][j][0] = (w0[j] << 4) & 0xF0F0F0F0u;
                  a[t][j][1] = (w1[j] << 4) & 0xF0F0F0F0u;
                  a[t][j][2] = w0[j] & 0xF0F0F0F0u;
                  a[t][j][3] = w1[j] & 0xF0F0F0F0u;
                }
              }
            }
            float sal[kTiles], sbl[kTiles];
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
              sal[t] = sa[t] * lane_mul;  // exact: a power of two
              sbl[t] = sb[t] * lane_mul;
            }
#pragma unroll
            for (int nt = 0; nt < NP; ++nt) {
              const uint4 b01 = kHoist ? hb01[kHoist ? nt : 0] : ptx::lds128(st + bofs[0] + nt * kDigitTile);
              const uint4 b23 = kHoist ? hb23[kHoist ? nt : 0] : ptx::lds128(st + bofs[1] + nt * kDigitTile);
              const float fct = kHoist ? hfct[kHoist ? nt : 0] : __uint_as_float(ptx::lds32(st + fofs + nt * 8));
              const int csum = kAsymSums ? static_cast<int>(ptx::lds32(st + sumofs + nt * 16)) : 0;
#pragma unroll
              for (int t = 0; t < kTiles; ++t) {
                int acc[4] = {0, 0, 0, 0};
                mma_s8(acc, a[t][0], b01.x, b01.y);
                mma_s8(acc, a[t][1], b01.z, b01.w);
                mma_s8(acc, a[t][2], b23.x, b23.y);
                mma_s8(acc, a[t][3], b23.z, b23.w);
                // Exact in int32: |q d| sums stay below 2^26, |z C| below 2^26.
                const float p0 = static_cast<float>(acc[0] + 256 * acc[1] -
                                                    (kAsymSums ? static_cast<int>(za[t]) * csum : 0));
                const float p1 = static_cast<float>(acc[2] + 256 * acc[3] -
                                                    (kAsymSums ? static_cast<int>(zb[t]) * csum : 0));
                tot[t][nt][0] = fmaf(p0 * fct, sal[t], tot[t][nt][0]);
                tot[t][nt][1] = fmaf(p1 * fct, sbl[t], tot[t][nt][1]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&empty[s]));
      }
      // Segment end: lane sums of both K slots, each output the sum of its
      // even (P01) and odd (P23) lane, in a fixed order.
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NP; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            red[(((cw * kTiles + t) * NP + nt) * 2 + h) * 32 + lane] = tot[t][nt][h];
      const bool stop = ptx::bar_red_or(1, kConsumers * 32, !ok || *abort_flag != 0u);
      const bool whole = (blo == 0 && bhi == KB);
      if (!stop) {
        float* dst = whole ? nullptr
                           : partials + (2 * static_cast<int64_t>(blockIdx.x) + (blo == 0 ? 1 : 0)) * kOut;
        for (int e = threadIdx.x - 32; e < kOut; e += kConsumers * 32) {
          const int mp = e & 1, gq = (e >> 1) & 7, hh = (e >> 4) & 1, rest = e >> 5;
          const int nt = rest % NP, tw = rest / NP;
          const int base = ((tw * NP + nt) * 2 + hh) * 32 + 4 * gq + 2 * mp;
          float sum = 0.0f;
#pragma unroll
          for (int q = 0; q < kSK; ++q) sum += red[q * S::kRedPer + base] + red[q * S::kRedPer + base + 1];
          if (!whole) {
            dst[e] = sum;
            continue;
          }
          const int m = 2 * nt + mp;
          const int64_t row = row0 + tw * 16 + tile_row<1>(gq) + 8 * hh;
          if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
        }
      }
      ptx::bar_sync(1, kConsumers * 32);
      if (stop) break;
      if (!whole) {
        const int64_t t0 = r * KB, t1 = (r + 1) * KB;
        const int p_first = static_cast<int>(((t0 + 1) * P + U - 1) / U - 1);
        const int p_last = static_cast<int>((t1 * P + U - 1) / U - 1);
        if (cw == 0 && lane == 0) {
          // The barrier above orders the CTA's partial stores before this
          // fence; fence and count release them to the last contributor.
          __threadfence();
          const uint32_t before = atomicAdd(&counters[p_first], 1u);
          const bool last = before == static_cast<uint32_t>(p_last - p_first);
          if (last) __threadfence();
          *last_flag = last ? 1u : 0u;
        }
        ptx::bar_sync(1, kConsumers * 32);
        if (*last_flag) {
          const float* first = partials + (2 * static_cast<int64_t>(p_first) + 1) * kOut;
          const float* rest = partials + 2 * static_cast<int64_t>(p_first + 1) * kOut;
          const int n_rest = p_last - p_first;
          for (int e = threadIdx.x - 32; e < kOut; e += kConsumers * 32) {
            float sum = __ldcg(first + e);
            for (int q = 0; q < n_rest; ++q) sum += __ldcg(rest + static_cast<int64_t>(2 * q) * kOut + e);
            const int mp = e & 1, gq = (e >> 1) & 7, hh = (e >> 4) & 1, rest_i = e >> 5;
            const int m = 2 * (rest_i % NP) + mp;
            const int tw = rest_i / NP;
            const int64_t row = row0 + tw * 16 + tile_row<1>(gq) + 8 * hh;
            if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
          }
          if (cw == 0 && lane == 0) counters[p_first] = 0u;
        }
      }
      u = r * KB + bhi;
    }
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

// ---------------- small matrices ----------------
// Decode for matrices whose 16-row tiles fit one wave: one CTA per tile,
// kSmallWarps warps splitting K (warp w takes 128-k blocks w, w + 8, ...,
// two at a time for M <= 8).  A lane loads its weight words and x fragments straight
// from global memory with 128-bit loads, expands and multiplies them exactly
// as the pipelined kernel does, and scales each block by its group's scale;
// the warps' partial sums are added in warp order through shared memory.  No
// copy engine, barrier ring or scratch: the pipelined kernel's fixed latency
// dominates at these sizes.
constexpr int kSmallWarps = 8;
constexpr int kSmallCtasPerSm = 3;

template <typename TX, int NT, bool ASYM>
__global__ void __launch_bounds__(kSmallWarps * 32, kSmallCtasPerSm) decode_small_kernel(
    const TX* __restrict__ x, const uint8_t* __restrict__ packed, const uint16_t* __restrict__ scales,
    const uint8_t* __restrict__ zeros, Epilogue ep, float* __restrict__ y, int64_t K, int group,
    int G, int M, int64_t N, int KB) {
  __shared__ float red[kSmallWarps * NT * 4 * 32];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int64_t ra = (row0 + g < N) ? row0 + g : N - 1;          // loads stay in bounds
  const int64_t rb = (row0 + g + 8 < N) ? row0 + g + 8 : N - 1;
  const int64_t Kp = K / 2;
  const uint8_t* wa = packed + ra * Kp + 16 * c;
  const uint8_t* wb = packed + rb * Kp + 16 * c;
  const uint16_t* sa_row = scales + ra * G;
  const uint16_t* sb_row = scales + rb * G;
  const uint8_t* za_row = ASYM ? zeros + ra * G : nullptr;
  const uint8_t* zb_row = ASYM ? zeros + rb * G : nullptr;
  // Launched as a programmatic dependent of what precedes it on the stream:
  // ask L2 for the weight lines of this warp's first step (L2 is coherent, so
  // lines the earlier kernel still writes are read fresh after the wait), let
  // the next kernel start its own set-up, then wait for the earlier kernel
  // before reading any input or writing y.
  if (warp < KB) {
    ptx::prefetch_l2(wa + static_cast<int64_t>(warp) * 64);
    ptx::prefetch_l2(wb + static_cast<int64_t>(warp) * 64);
  }
  ptx::launch_dependents();
  ptx::grid_dependency_wait();
  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) tot[nt][i] = 0.0f;
  constexpr int kStep = NT == 1 ? 2 : 1;  // blocks per step (x fragments of M > 8 take twice the registers)
  for (int kb0 = warp; kb0 < KB; kb0 += kStep * kSmallWarps) {
    // kStep blocks per step, all loads issued before any use.
    uint4 ua[kStep], ub[kStep], xf4[kStep][4][NT];
    uint32_t sraw[kStep][2];
    uint32_t zraw[kStep][2];
#pragma unroll
    for (int q = 0; q < kStep; ++q) {
      const int kb = kb0 + kSmallWarps * q;
      const bool ok = kb < KB;
      const int kc = ok ? kb : kb0;
      ua[q] = __ldg(reinterpret_cast<const uint4*>(wa + static_cast<int64_t>(kc) * 64));
      ub[q] = __ldg(reinterpret_cast<const uint4*>(wb + static_cast<int64_t>(kc) * 64));
      const int gi = static_cast<int>(static_cast<int64_t>(kc) * 128 / group);
      sraw[q][0] = __ldg(sa_row + gi);
      sraw[q][1] = __ldg(sb_row + gi);
      zraw[q][0] = ASYM ? __ldg(za_row + gi) : 0u;
      zraw[q][1] = ASYM ? __ldg(zb_row + gi) : 0u;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = g + 8 * nt;
        const TX* xp = x + static_cast<int64_t>(n < M ? n : 0) * K + static_cast<int64_t>(kc) * 128 + 32 * c;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xf4[q][j][nt] = (n < M) ? __ldg(reinterpret_cast<const uint4*>(xp + 8 * j)) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int q = 0; q < kStep; ++q) {
      if (kb0 + kSmallWarps * q >= KB) break;
      const uint32_t wva[4] = {ua[q].x, ua[q].y, ua[q].z, ua[q].w};
      const uint32_t wvb[4] = {ub[q].x, ub[q].y, ub[q].z, ub[q].w};
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
      const uint32_t zba = ASYM ? Cvt<TX>::zero_bias(zraw[q][0]) : Cvt<TX>::kMagic;
      const uint32_t zbb = ASYM ? Cvt<TX>::zero_bias(zraw[q][1]) : Cvt<TX>::kMagic;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pa[4], pb[4];
        expand<TX, ASYM>(wva[j], pa, zba);
        expand<TX, ASYM>(wvb[j], pb, zbb);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 xf = pair_x(xf4[q][j][nt]);
          Cvt<TX>::mma(acc[nt], pa[0], pb[0], pa[1], pb[1], xf.x, xf.y);
          Cvt<TX>::mma(acc[nt], pa[2], pb[2], pa[3], pb[3], xf.z, xf.w);
        }
      }
      const float sa = f16_bits_to_float(sraw[q][0]);
      const float sb = f16_bits_to_float(sraw[q][1]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        tot[nt][0] = fmaf(acc[nt][0], sa, tot[nt][0]);
        tot[nt][1] = fmaf(acc[nt][1], sa, tot[nt][1]);
        tot[nt][2] = fmaf(acc[nt][2], sb, tot[nt][2]);
        tot[nt][3] = fmaf(acc[nt][3], sb, tot[nt][3]);
      }
    }
  }
  // Warps' partials summed in warp order.
  constexpr int kPerWarp = NT * 4 * 32;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp * kPerWarp + (nt * 4 + i) * 32 + lane] = tot[nt][i];
  __syncthreads();
  for (int e = threadIdx.x; e < kPerWarp; e += blockDim.x) {
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) sum += red[w * kPerWarp + e];
    const int ln = e & 31;
    const int i = (e >> 5) & 3;
    const int nt = e >> 7;
    const int m = nt * 8 + 2 * (ln & 3) + (i & 1);
    const int64_t row = row0 + (ln >> 2) + ((i < 2) ? 0 : 8);
    if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
  }
}

template <typename TX, bool ASYM>
cudaError_t launch_small(const TX* x, const uint8_t* packed, const uint16_t* scales,
                         const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                         int64_t N, float* y, cudaStream_t stream) {
  const int G = static_cast<int>((K + group - 1) / group);
  const int KB = static_cast<int>((K + 127) / 128);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + 15) / 16));
  cfg.blockDim = dim3(kSmallWarps * 32);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (M <= 8)
    return cudaLaunchKernelEx(&cfg, decode_small_kernel<TX, 1, ASYM>, x, packed, scales, zeros, ep,
                              y, K, group, G, static_cast<int>(M), N, KB);
  return cudaLaunchKernelEx(&cfg, decode_small_kernel<TX, 2, ASYM>, x, packed, scales, zeros, ep, y,
                            K, group, G, static_cast<int>(M), N, KB);
}

// Small matrices: 16-row tiles that fit one wave, K a multiple of 128 (so
// every block is whole) and groups of whole blocks.
bool small_applies(int64_t K, int group, int64_t N) {
  if (!INT4_DECODE_SMALL || group % 128 != 0 || K % 128 != 0) return false;
  return (N + 15) / 16 <= static_cast<int64_t>(kSmallCtasPerSm) * num_sms();
}

// ---------------- matrices that fit in shared memory ----------------
// Decode for matrices whose 16-row tiles all fit in shared memory at once
// (one wave, each tile's packed rows resident in its CTA): right after the
// dependency wait, every CTA issues bulk copies of its whole tile (row by
// row, in chunks of kFlatChunk bytes of each row, one barrier per chunk) and,
// for M <= 2 when it fits, of x, and loads the tile's scales into shared
// memory, so the whole matrix is requested in one round trip and the loop
// over K reads shared memory only.  W warps split K as in
// decode_small_kernel (warp w takes 128-k blocks w, w + W, ...), with the
// small kernel's arithmetic per block; the warps' partials are added in warp
// order.
#ifndef INT4_FLAT_PDL_LATE
#define INT4_FLAT_PDL_LATE 1  // let the next kernel launch only after this CTA's loop
#endif
#ifndef INT4_FLAT_CHUNK
#define INT4_FLAT_CHUNK 2048
#endif
constexpr int kFlatChunk = INT4_FLAT_CHUNK;  // bytes of each row per copy chunk (a multiple of 64)

// Row stride of the resident tile: Kp (a multiple of 64) padded so that the
// lanes of one shared-memory wavefront hit distinct banks: the row stride in
// words is 16, 8 or 4 modulo 32 for the 16-, 8- and 4-byte weight loads of
// groups of whole blocks, of 64 and of 32 (GPB = 1, 2, 4 groups per block).
__host__ __device__ constexpr int64_t flat_row_stride(int64_t Kp, int gpb) {
  return Kp + ((128 + 64 / gpb) - Kp % 128) % 128;
}

// Shared-memory layout of a CTA: the tile's rows, x (if staged), the tile's
// scales [16, G] (and zero points), the barriers (chunks, then x).
struct FlatLayout {
  int64_t rstride, off_x, off_s, off_z, off_bar, bytes;
  int nch;
};
__host__ __device__ inline FlatLayout flat_layout(int64_t K, int G, int M, bool xs, bool asym, int gpb) {
  FlatLayout L;
  const int64_t Kp = K / 2;
  L.rstride = flat_row_stride(Kp, gpb);
  L.nch = static_cast<int>((Kp + kFlatChunk - 1) / kFlatChunk);
  L.off_x = 16 * L.rstride;
  L.off_s = L.off_x + (xs ? static_cast<int64_t>(M) * K * 2 : 0);
  L.off_z = L.off_s + (16 * static_cast<int64_t>(G) * 2 + 15) / 16 * 16;
  L.off_bar = L.off_z + (asym ? (16 * static_cast<int64_t>(G) + 15) / 16 * 16 : 0);
  L.bytes = L.off_bar + 8 * (L.nch + 1);
  return L;
}

template <typename TX, int NT, bool ASYM, int W, bool XS, int GPB>
__global__ void __launch_bounds__(W * 32, W == 8 ? 2 : 5) decode_flat_kernel(
    const TX* __restrict__ x, const uint8_t* __restrict__ packed, const uint16_t* __restrict__ scales,
    const uint8_t* __restrict__ zeros, Epilogue ep, float* __restrict__ y, int64_t K, int group,
    int G, int M, int64_t N, int KB, uint32_t* status) {
  static_assert(!XS || NT == 1, "x is staged for M <= 2 only");
  extern __shared__ __align__(16) uint8_t tile_smem[];
  __shared__ float red[W * NT * 4 * 32];
  __shared__ uint32_t abort_word;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t Kp = K / 2;
  const FlatLayout L = flat_layout(K, G, M, XS, ASYM, GPB);
  const int nch = L.nch;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tile_smem + L.off_bar);  // chunks, then x
  const uint32_t tbase = ptx::smem_u32(tile_smem);
  uint16_t* s_sc = reinterpret_cast<uint16_t*>(tile_smem + L.off_s);
  uint8_t* s_z = tile_smem + L.off_z;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int rows = static_cast<int>(N - row0 < 16 ? N - row0 : 16);
  const WaitCtx wc{&abort_word, status};
  if (threadIdx.x == 0) {
    for (int i = 0; i < nch + (XS ? 1 : 0); ++i) ptx::mbar_init(ptx::smem_u32(&bars[i]), 1);
    abort_word = 0u;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // Launched as a programmatic dependent of what precedes it on the stream:
  // the set-up above overlaps that kernel's tail; nothing is read before the
  // wait.  The next kernel is let in only after this CTA's loop: its CTAs,
  // small enough to sit beside these ones while they wait for this grid,
  // took issue slots from the loop (4096 x 4096 at M = 1: 8.3 against
  // 6.2 us per call back to back).
  if (!INT4_FLAT_PDL_LATE) ptx::launch_dependents();
  ptx::grid_dependency_wait();
  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nch; ++i) {
        const int64_t off = static_cast<int64_t>(i) * kFlatChunk;
        const int64_t cb = Kp - off < kFlatChunk ? Kp - off : kFlatChunk;
        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&bars[i]), static_cast<uint32_t>(rows * cb));
      }
      if (XS) {
        const uint32_t xb = static_cast<uint32_t>(static_cast<int64_t>(M) * K * 2);
        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&bars[nch]), xb);
        ptx::bulk_load(tbase + static_cast<uint32_t>(L.off_x), x, xb, ptx::smem_u32(&bars[nch]));
      }
    }
    __syncwarp();
    // Chunk-major order: every row's first chunk is requested first.
    for (int i = lane; i < rows * nch; i += 32) {
      const int r = i % rows, ch = i / rows;
      const int64_t off = static_cast<int64_t>(ch) * kFlatChunk;
      const int64_t cb = Kp - off < kFlatChunk ? Kp - off : kFlatChunk;
      ptx::bulk_load(tbase + static_cast<uint32_t>(r * L.rstride + off), packed + (row0 + r) * Kp + off,
                     static_cast<uint32_t>(cb), ptx::smem_u32(&bars[ch]));
    }
  }
  // The tile's scales (and zero points): rows*G contiguous values.
  for (int i = threadIdx.x; i < rows * G; i += blockDim.x) {
    s_sc[i] = __ldg(scales + row0 * G + i);
    if (ASYM) s_z[i] = __ldg(zeros + row0 * G + i);
  }
  __syncthreads();
  // Rows past N are never copied; their (stale) words and scales only reach
  // outputs that are not stored.
  // Lane (g, c) reads words word_index<GPB>(c, j), j = 0..3, of rows g and
  // g + 8 of each block, so that word j of the four lanes of a quad lies in
  // one group; its x fragments are the same words of x.
  const uint32_t wa = tbase + static_cast<uint32_t>(g * L.rstride);
  const uint32_t wb = tbase + static_cast<uint32_t>((g + 8) * L.rstride);
  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) tot[nt][i] = 0.0f;
  // x fragments of block kb from global memory (L2-resident), one block ahead.
  auto load_x = [&](int kb, uint4 (&xf)[4][NT]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = g + 8 * nt;
      const TX* xp = x + static_cast<int64_t>(n < M ? n : 0) * K + static_cast<int64_t>(kb) * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        xf[j][nt] = (n < M) ? __ldg(reinterpret_cast<const uint4*>(xp + 8 * word_index<GPB>(c, j)))
                            : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 xc[4][NT], xn[4][NT];
  bool ok = true;
  if (XS) {
    ok = __all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&bars[nch]), 0u, wc));
  } else if (warp < KB) {
    load_x(warp, xc);
  }
  const int n0 = g < M ? g : 0;  // staged x: this lane's batch row
  for (int kb = warp; ok && kb < KB; kb += W) {
    if (XS) {
      const uint32_t xs = tbase + static_cast<uint32_t>(L.off_x + (static_cast<int64_t>(n0) * K + kb * 128) * 2);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        xc[j][0] = g < M ? ptx::lds128(xs + 16 * word_index<GPB>(c, j)) : make_uint4(0u, 0u, 0u, 0u);
    } else if (kb + W < KB) {
      load_x(kb + W, xn);
    }
    const int ch = (kb * 64) / kFlatChunk;
    ok = __all_sync(0xffffffffu, wait_bar(ptx::smem_u32(&bars[ch]), 0u, wc));
    if (!ok) break;
    uint32_t wva[4], wvb[4];
    if (GPB == 1) {
      const uint4 ua = ptx::lds128(wa + kb * 64 + 16 * c);
      const uint4 ub = ptx::lds128(wb + kb * 64 + 16 * c);
      wva[0] = ua.x; wva[1] = ua.y; wva[2] = ua.z; wva[3] = ua.w;
      wvb[0] = ub.x; wvb[1] = ub.y; wvb[2] = ub.z; wvb[3] = ub.w;
    } else if (GPB == 2) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 ua = ptx::lds64(wa + kb * 64 + 4 * (8 * h + 2 * c));
        const uint2 ub = ptx::lds64(wb + kb * 64 + 4 * (8 * h + 2 * c));
        wva[2 * h] = ua.x; wva[2 * h + 1] = ua.y;
        wvb[2 * h] = ub.x; wvb[2 * h + 1] = ub.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wva[j] = ptx::lds32(wa + kb * 64 + 4 * (4 * j + c));
        wvb[j] = ptx::lds32(wb + kb * 64 + 4 * (4 * j + c));
      }
    }
    // One accumulator per group of the block (GPB of them), each scaled by
    // its group's scale and added in order.
    constexpr int kJPer = 4 / GPB;  // words j per group
#pragma unroll
    for (int sg = 0; sg < GPB; ++sg) {
      const int gi = GPB == 1 ? static_cast<int>(static_cast<int64_t>(kb) * 128 / group) : kb * GPB + sg;
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
      const uint32_t zba = ASYM ? Cvt<TX>::zero_bias(s_z[g * G + gi]) : Cvt<TX>::kMagic;
      const uint32_t zbb = ASYM ? Cvt<TX>::zero_bias(s_z[(g + 8) * G + gi]) : Cvt<TX>::kMagic;
#pragma unroll
      for (int jj = 0; jj < kJPer; ++jj) {
        const int j = sg * kJPer + jj;
        uint32_t pa[4], pb[4];
        expand<TX, ASYM>(wva[j], pa, zba);
        expand<TX, ASYM>(wvb[j], pb, zbb);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 xf = pair_x(xc[j][nt]);
          Cvt<TX>::mma(acc[nt], pa[0], pb[0], pa[1], pb[1], xf.x, xf.y);
          Cvt<TX>::mma(acc[nt], pa[2], pb[2], pa[3], pb[3], xf.z, xf.w);
        }
      }
      const float sa = f16_bits_to_float(s_sc[g * G + gi]);
      const float sb = f16_bits_to_float(s_sc[(g + 8) * G + gi]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        tot[nt][0] = fmaf(acc[nt][0], sa, tot[nt][0]);
        tot[nt][1] = fmaf(acc[nt][1], sa, tot[nt][1]);
        tot[nt][2] = fmaf(acc[nt][2], sb, tot[nt][2]);
        tot[nt][3] = fmaf(acc[nt][3], sb, tot[nt][3]);
      }
    }
    if (!XS) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xc[j][nt] = xn[j][nt];
    }
  }
  if (INT4_FLAT_PDL_LATE) ptx::launch_dependents();
  // Warps' partials summed in warp order.
  constexpr int kPerWarp = NT * 4 * 32;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp * kPerWarp + (nt * 4 + i) * 32 + lane] = tot[nt][i];
  __syncthreads();
  if (abort_word != 0u) {
    // A wait gave up: let the copies in flight land before the CTA's
    // shared memory is released, and store nothing.
    if (threadIdx.x == 0)
      for (int i = 0; i < nch + (XS ? 1 : 0); ++i) drain_bar(ptx::smem_u32(&bars[i]), 0u);
    return;
  }
  for (int e = threadIdx.x; e < kPerWarp; e += blockDim.x) {
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) sum += red[w * kPerWarp + e];
    const int ln = e & 31;
    const int i = (e >> 5) & 3;
    const int nt = e >> 7;
    const int m = nt * 8 + 2 * (ln & 3) + (i & 1);
    const int64_t row = row0 + (ln >> 2) + ((i < 2) ? 0 : 8);
    if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = ep.apply(sum, row);
  }
}

// CTAs per SM of one shared-memory decode kernel for a layout of `bytes`
// bytes, queried once per device and size.
template <typename TX, int NT, bool ASYM, int W, bool XS, int GPB>
int flat_occupancy(int64_t bytes) {
  constexpr int kMaxDevices = 64;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  static thread_local int64_t last_bytes[kMaxDevices] = {};
  static thread_local int last_occ[kMaxDevices] = {};
  if (last_bytes[dev] == bytes) return last_occ[dev];
  int occ = 0;
  // The opt-in is the device's limit less the kernel's static shared memory,
  // the same for every shape, so concurrent callers agree.
  const void* fn = reinterpret_cast<const void*>(decode_flat_kernel<TX, NT, ASYM, W, XS, GPB>);
  int optin = 0;
  cudaFuncAttributes fa;
  bool failed = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
                cudaFuncGetAttributes(&fa, fn) != cudaSuccess;
  if (!failed) {
    const int64_t max_dyn = static_cast<int64_t>(optin) - static_cast<int64_t>(fa.sharedSizeBytes);
    if (bytes <= max_dyn)
      failed = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(max_dyn)) !=
                   cudaSuccess ||
               cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, W * 32, static_cast<size_t>(bytes)) !=
                   cudaSuccess;
  }
  if (failed) {
    occ = 0;
    (void)cudaGetLastError();  // a refused query only rules this kernel out
  }
  last_bytes[dev] = bytes;
  last_occ[dev] = occ;
  return occ;
}

// Kernel choice for a shape: warps per CTA (8, else 4) and whether x is
// staged (M <= 2, preferred), the first whose tiles fit one wave; 0 when
// none does (the shape then takes another decode kernel).
constexpr int kFlatXs = 0x100;

template <typename TX, int NT, bool ASYM, int W, bool XS, int GPB>
bool flat_fits(int64_t K, int G, int M, int64_t tiles) {
  const int64_t bytes = flat_layout(K, G, M, XS, ASYM, GPB).bytes;
  return tiles <= static_cast<int64_t>(flat_occupancy<TX, NT, ASYM, W, XS, GPB>(bytes)) * num_sms();
}

template <typename TX, bool ASYM, int GPB>
int flat_choice_g(int64_t K, int G, int m, int64_t tiles) {
  if (m <= 8) {
    if (m <= 2 && flat_fits<TX, 1, ASYM, 8, true, GPB>(K, G, m, tiles)) return 8 | kFlatXs;
    if (flat_fits<TX, 1, ASYM, 8, false, GPB>(K, G, m, tiles)) return 8;
    if (m <= 2 && flat_fits<TX, 1, ASYM, 4, true, GPB>(K, G, m, tiles)) return 4 | kFlatXs;
    if (flat_fits<TX, 1, ASYM, 4, false, GPB>(K, G, m, tiles)) return 4;
    return 0;
  }
  if (flat_fits<TX, 2, ASYM, 8, false, GPB>(K, G, m, tiles)) return 8;
  // Four warps with a group per word at M > 8 spill, and lose to the
  // pipelined 16-bit kernel (W [11008, 4096], group 32, M = 16: 25.3
  // against 22.2 us).
  if constexpr (GPB == 1) {
    if (flat_fits<TX, 2, ASYM, 4, false, GPB>(K, G, m, tiles)) return 4;
  }
  return 0;
}

template <typename TX, bool ASYM>
int flat_choice(int64_t K, int group, int64_t M, int64_t N) {
  if (!INT4_DECODE_FLAT || K % 128 != 0 || M > 16) return 0;
  if (!(group == 32 || group == 64 || group % 128 == 0)) return 0;
  // Where the integer kernel would convert x inside its CTAs (M <= 2 on a
  // matrix too tall for the small-matrix kernel), it is faster: its
  // arithmetic takes a quarter of the instructions per weight.
  if (group % 128 == 0 && M <= kFuseMaxM && !small_applies(K, group, N)) return 0;
  const int G = static_cast<int>(K / group + (K % group != 0));
  const int64_t tiles = (N + 15) / 16;
  const int m = static_cast<int>(M);
  const int gpb = group == 32 ? 4 : group == 64 ? 2 : 1;
  const int c = gpb == 4   ? flat_choice_g<TX, ASYM, 4>(K, G, m, tiles)
                : gpb == 2 ? flat_choice_g<TX, ASYM, 2>(K, G, m, tiles)
                           : flat_choice_g<TX, ASYM, 1>(K, G, m, tiles);
  return c == 0 ? 0 : c | (gpb << 12);
}

template <typename TX, int NT, bool ASYM, int W, bool XS, int GPB>
cudaError_t launch_flat_w(const TX* x, const uint8_t* packed, const uint16_t* scales,
                          const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                          int64_t N, float* y, cudaStream_t stream) {
  uint32_t* status = status_word();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  const int G = static_cast<int>((K + group - 1) / group);
  const int KB = static_cast<int>((K + 127) / 128);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + 15) / 16));
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(flat_layout(K, G, static_cast<int>(M), XS, ASYM, GPB).bytes);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_flat_kernel<TX, NT, ASYM, W, XS, GPB>, x, packed, scales, zeros, ep,
                            y, K, group, G, static_cast<int>(M), N, KB, status);
}

template <typename TX, bool ASYM, int GPB>
cudaError_t launch_flat_g(int choice, const TX* x, const uint8_t* packed, const uint16_t* scales,
                          const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                          int64_t N, float* y, cudaStream_t stream) {
  const bool xs = (choice & kFlatXs) != 0;
  const int w = choice & 0xFF;
  if (M <= 8) {
    if (w == 8)
      return xs ? launch_flat_w<TX, 1, ASYM, 8, true, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream)
                : launch_flat_w<TX, 1, ASYM, 8, false, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream);
    return xs ? launch_flat_w<TX, 1, ASYM, 4, true, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream)
              : launch_flat_w<TX, 1, ASYM, 4, false, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream);
  }
  if constexpr (GPB == 1) {
    if (w == 4)
      return launch_flat_w<TX, 2, ASYM, 4, false, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream);
  }
  // (flat_choice picks 4 warps at M > 8 only for groups of whole blocks.)
  return launch_flat_w<TX, 2, ASYM, 8, false, GPB>(x, packed, scales, zeros, ep, K, group, M, N, y, stream);
}

// `choice`: flat_choice's value (warps, staged x, groups per block in bits 12+).
template <typename TX, bool ASYM>
cudaError_t launch_flat(int choice, const TX* x, const uint8_t* packed, const uint16_t* scales,
                        const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                        int64_t N, float* y, cudaStream_t stream) {
  const int gpb = choice >> 12;
  if (gpb == 4) return launch_flat_g<TX, ASYM, 4>(choice, x, packed, scales, zeros, ep, K, group, M, N, y, stream);
  if (gpb == 2) return launch_flat_g<TX, ASYM, 2>(choice, x, packed, scales, zeros, ep, K, group, M, N, y, stream);
  return launch_flat_g<TX, ASYM, 1>(choice, x, packed, scales, zeros, ep, K, group, M, N, y, stream);
}

// ---------------- host side: scratch, schedule, launch ----------------
// A decode call may need device scratch: one arrival counter per CTA (zero
// when the call starts; every call leaves its counters zero), two partial-
// tile slots per CTA for the split, and the x digit records of the integer
// kernel at M > 2.  The caller provides it (int4_matmul_ws), or it is the
// library's fixed array (int4_matmul_decode_noalloc).  Without any
// (int4_matmul), the runs cover whole row tiles, so no tile is split, and
// batches that would need digit records take the 16-bit kernel.
struct DecodeScratch {
  uint32_t* counters = nullptr;
  size_t counter_cap = 0;  // entries
  float* partials = nullptr;
  size_t partial_cap = 0;  // floats
  uint8_t* records = nullptr;
  size_t record_cap = 0;   // bytes
};

struct DecodeNeed {
  size_t counters = 0;  // entries
  size_t partials = 0;  // floats
  size_t records = 0;   // bytes
};

// A caller's workspace: the counters in a fixed first region (so that calls
// of any shape sharing the workspace find zeros there), then the partial
// tiles, then the records, each region 256-byte aligned.
constexpr size_t kWsCounterCap = 1024;
constexpr size_t kWsCounterBytes = kWsCounterCap * sizeof(uint32_t);

size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

size_t workspace_bytes(const DecodeNeed& n) {
  if (n.counters == 0 && n.partials == 0 && n.records == 0) return 0;
  return kWsCounterBytes + round256(n.partials * sizeof(float)) + n.records;
}

DecodeScratch carve_workspace(void* ws, const DecodeNeed& n) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  DecodeScratch s;
  s.counters = reinterpret_cast<uint32_t*>(b);
  s.counter_cap = kWsCounterCap;
  s.partials = reinterpret_cast<float*>(b + kWsCounterBytes);
  s.partial_cap = n.partials;
  s.records = b + kWsCounterBytes + round256(n.partials * sizeof(float));
  s.record_cap = n.records;
  return s;
}

// Scratch of int4_matmul_decode_noalloc: partial slots, arrival counters and
// the x digit records in one fixed device array (zero at load; every call
// leaves the counters zero).  4 MiB of partials hold one wave of up to 512
// CTAs (B200 runs 296: 2 per SM); 4 MiB of records hold K up to 64384 at
// M = 16 (246528 at M <= 4; M <= 2 converts x in the matmul and needs none).
constexpr int kNoAllocMaxCtas = 512;
constexpr size_t kNoAllocPartialBytes = size_t(4) << 20;
constexpr size_t kNoAllocCounterBytes = kNoAllocMaxCtas * sizeof(uint32_t);
constexpr size_t kNoAllocRecordBytes = size_t(4) << 20;  // x digit records
constexpr size_t kNoAllocScratchBytes = kNoAllocPartialBytes + kNoAllocCounterBytes + kNoAllocRecordBytes;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of the array on the current device, resolved once per
// device with cudaGetSymbolAddress (no allocation).
cudaError_t noalloc_scratch(float** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static float* cache[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    cache[dev] = static_cast<float*>(p);
  }
  *out = cache[dev];
  return cudaSuccess;
}

// The array's regions as a scratch descriptor.
DecodeScratch noalloc_regions(float* base) {
  char* b = reinterpret_cast<char*>(base);
  DecodeScratch s;
  s.partials = base;
  s.partial_cap = kNoAllocPartialBytes / sizeof(float);
  s.counters = reinterpret_cast<uint32_t*>(b + kNoAllocPartialBytes);
  s.counter_cap = kNoAllocMaxCtas;
  s.records = reinterpret_cast<uint8_t*>(b + kNoAllocPartialBytes + kNoAllocCounterBytes);
  s.record_cap = kNoAllocRecordBytes;
  return s;
}

// Grid and runs of one decode call: P CTAs (one wave at the occupancy limit,
// at most one per counter of the workspace layout), each with an equal run
// of (row tile, K block) units whose ends fall on multiples of `gran`.
struct DecodePlan {
  int KB = 0;
  int64_t U = 0;
  int64_t P = 0;
  int64_t gran = 1;
  bool split = false;  // does some run start or end inside a tile?
};

// Shared-memory opt-in and occupancy of a decode kernel, once per device.
cudaError_t kernel_occupancy(const void* fn, int threads, int alloc, std::atomic<int>* cache,
                             int* occ_out) {
  constexpr int kMaxDevices = 64;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int occ = cache[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, alloc);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, alloc);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    cache[dev].store(occ, std::memory_order_relaxed);
  }
  *occ_out = occ;
  return cudaSuccess;
}

// The runs for `occ` CTAs per SM over row tiles of `rows` rows: equal runs
// of blocks (the split) when scratch holds the partial tiles, else runs of
// whole tiles.
void plan_runs(int occ, int rows, int64_t K, int64_t N, bool may_split, DecodePlan* pl) {
  pl->KB = static_cast<int>((K + 127) / 128);
  const int64_t tiles = (N + rows - 1) / rows;
  pl->U = tiles * pl->KB;
  int64_t slots = static_cast<int64_t>(occ) * num_sms();
  if (slots > static_cast<int64_t>(kWsCounterCap)) slots = kWsCounterCap;
  if (!may_split) {
    pl->gran = pl->KB;
    pl->P = slots < tiles ? slots : tiles;
    pl->split = false;
    return;
  }
  pl->gran = 1;
  pl->P = slots < pl->U ? slots : pl->U;
  // Remembered for the last shape seen by this thread: the scan costs a
  // division per CTA.
  thread_local int64_t last_U = -1, last_P = -1, last_KB = -1;
  thread_local bool last_split = false;
  if (pl->U != last_U || pl->P != last_P || pl->KB != last_KB) {
    bool sp = false;
    for (int64_t p = 1; p < pl->P && !sp; ++p) sp = (p * pl->U / pl->P) % pl->KB != 0;
    last_U = pl->U;
    last_P = pl->P;
    last_KB = pl->KB;
    last_split = sp;
  }
  pl->split = last_split;
}

// Arguments of one decode call (zeros: the asymmetric scheme's zero points,
// or nullptr for the symmetric scheme).
struct DecodeArgs {
  const void* x;
  const uint8_t* packed;
  const uint16_t* scales;
  const uint8_t* zeros;
  Epilogue ep;
  int64_t K;
  int group;
  int64_t M;
  int64_t N;
  float* y;
  cudaStream_t stream;
};

bool fits(const DecodeNeed& n, const DecodeScratch* sc) {
  if (n.counters == 0 && n.partials == 0 && n.records == 0) return true;
  return sc != nullptr && n.counters <= sc->counter_cap && n.partials <= sc->partial_cap &&
         n.records <= sc->record_cap;
}

template <typename TX, int NT, int GPB, bool ASYM>
cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& pl, float* partials,
                          uint32_t* counters) {
  using L = DLayout<NT>;
  constexpr int kRowsPerCta = Tiles<NT>::kRowsPerCta;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  uint32_t* status = status_word();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  const int G = static_cast<int>((a.K + a.group - 1) / a.group);
  CUtensorMap tw, tx;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 2), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 2)};
    const cuuint32_t box[2] = {128, kRowsPerCta};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K) * 2};
    const cuuint32_t box[2] = {256, static_cast<cuuint32_t>(a.M)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = std::is_same<TX, __nv_bfloat16>::value
                                       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (enc(&tx, dt, 2, const_cast<void*>(a.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.P));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = a.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<TX, NT, GPB, ASYM>, tw, tx, a.scales, a.zeros, a.ep,
                            a.y, a.K, a.group, G, static_cast<int>(a.M), a.N, pl.KB, pl.U,
                            static_cast<int>(pl.P), pl.gran, partials, counters, status);
}

// The 16-bit decode kernel: plan, scratch need and (if `launch`) the launch.
template <typename TX, int NT, int GPB, bool ASYM>
cudaError_t run_bf(const DecodeArgs& a, bool scratch, const DecodeScratch* sc, DecodeNeed* need,
                   bool launch) {
  constexpr int kPer = kRowGroups * Tiles<NT>::kTiles * NT * 4 * 32;  // outputs of a tile
  static std::atomic<int> occ_cache[64];
  int occ = 0;
  cudaError_t e = kernel_occupancy(reinterpret_cast<const void*>(decode_kernel<TX, NT, GPB, ASYM>),
                                   kThreads, DLayout<NT>::kAlloc, occ_cache, &occ);
  if (e != cudaSuccess) return e;
  DecodePlan pl;
  plan_runs(occ, Tiles<NT>::kRowsPerCta, a.K, a.N, scratch, &pl);
  DecodeNeed n;
  if (pl.split) {
    n.counters = static_cast<size_t>(pl.P);
    n.partials = static_cast<size_t>(2 * pl.P) * kPer;
  }
  *need = n;
  if (!launch) return cudaSuccess;
  if (!fits(n, sc)) return cudaErrorInvalidValue;
  return launch_decode<TX, NT, GPB, ASYM>(a, pl, pl.split ? sc->partials : nullptr,
                                    pl.split ? sc->counters : nullptr);
}

template <typename TX, int NP, bool FUSE, bool ASYM>
cudaError_t launch_decode_i8(const DecodeArgs& a, const DecodePlan& pl, float* partials,
                             uint32_t* counters, uint8_t* records) {
  using S = I8Shape<NP, FUSE>;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  uint32_t* status = status_word();
  if (status == nullptr) return cudaErrorInvalidSymbol;
  const TX* x = static_cast<const TX*>(a.x);
  const int G = static_cast<int>((a.K + a.group - 1) / a.group);
  CUtensorMap tw, tx;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 2), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 2)};
    const cuuint32_t box[2] = {128, S::kRowsPerCta};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.packed), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  std::memset(&tx, 0, sizeof tx);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  if (S::kFuse) {
    // x [M, K]: boxes of 256 k by all M rows.
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K) * 2};
    const cuuint32_t box[2] = {256, static_cast<cuuint32_t>(a.M)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = std::is_same<TX, __nv_bfloat16>::value
                                       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (enc(&tx, dt, 2, const_cast<TX*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // Records 0 .. KB: a stage whose second block is past the last reads the
    // zero record KB.
    const int64_t nrec = static_cast<int64_t>(pl.KB) + 1;
    const int MP = 2 * NP;
    const int64_t threads = 16 * MP * nrec;
    cudaLaunchConfig_t dcfg = {};
    dcfg.gridDim = dim3(static_cast<unsigned>((threads + 255) / 256));
    dcfg.blockDim = dim3(256);
    dcfg.stream = a.stream;
    dcfg.attrs = attr;
    dcfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&dcfg, x_digits_kernel<TX>, x, a.K,
                                             static_cast<int>(a.M), MP, NP, nrec, records);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.P));
  cfg.blockDim = dim3(S::kThreads);
  cfg.dynamicSmemBytes = S::kAlloc;
  cfg.stream = a.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_i8_kernel<TX, NP, FUSE, ASYM>, tw, tx, x,
                            static_cast<const uint8_t*>(records), a.scales, a.zeros, a.ep, a.y, a.K,
                            a.group, G,
                            static_cast<int>(a.M), a.N, pl.KB, pl.U, static_cast<int>(pl.P),
                            pl.gran, partials, counters, status);
}

// The integer decode kernel: plan, scratch need and (if `launch`) the launch.
template <typename TX, int NP, bool FUSE, bool ASYM>
cudaError_t run_i8(const DecodeArgs& a, bool scratch, const DecodeScratch* sc, DecodeNeed* need,
                   bool launch) {
  using S = I8Shape<NP, FUSE>;
  static std::atomic<int> occ_cache[64];
  int occ = 0;
  cudaError_t e = kernel_occupancy(reinterpret_cast<const void*>(decode_i8_kernel<TX, NP, FUSE, ASYM>),
                                   S::kThreads, S::kAlloc, occ_cache, &occ);
  if (e != cudaSuccess) return e;
  DecodePlan pl;
  plan_runs(occ, S::kRowsPerCta, a.K, a.N, scratch, &pl);
  DecodeNeed n;
  if (pl.split) {
    n.counters = static_cast<size_t>(pl.P);
    n.partials = static_cast<size_t>(2 * pl.P) * S::kOut;
  }
  if (!S::kFuse) n.records = static_cast<size_t>(pl.KB + 1) * S::kRec;
  *need = n;
  if (!launch) return cudaSuccess;
  if (!fits(n, sc)) return cudaErrorInvalidValue;
  return launch_decode_i8<TX, NP, FUSE, ASYM>(a, pl, pl.split ? sc->partials : nullptr,
                                        pl.split ? sc->counters : nullptr,
                                        S::kFuse ? nullptr : sc->records);
}

// Kernel choice of a decode call.  `scratch`: whether scratch will be there
// (the split schedule and, at M > 2 with groups of whole 128-k blocks, the
// integer kernel with digit records); without it the runs cover whole tiles
// and such batches take the 16-bit kernel.
template <typename TX, bool ASYM>
cudaError_t run_decode(const DecodeArgs& a, bool scratch, const DecodeScratch* sc, DecodeNeed* need,
                       bool launch) {
  if (const int fw = flat_choice<TX, ASYM>(a.K, a.group, a.M, a.N)) {
    *need = DecodeNeed{};
    if (!launch) return cudaSuccess;
    return launch_flat<TX, ASYM>(fw, static_cast<const TX*>(a.x), a.packed, a.scales, a.zeros, a.ep,
                                 a.K, a.group, a.M, a.N, a.y, a.stream);
  }
  if (small_applies(a.K, a.group, a.N)) {
    *need = DecodeNeed{};
    if (!launch) return cudaSuccess;
    return launch_small<TX, ASYM>(static_cast<const TX*>(a.x), a.packed, a.scales, a.zeros, a.ep,
                                  a.K, a.group, a.M, a.N, a.y, a.stream);
  }
  if (a.group % 128 == 0) {
    if (a.M <= kFuseMaxM) return run_i8<TX, 1, true, ASYM>(a, scratch, sc, need, launch);
    if (!scratch) {
      if (a.M <= 8) return run_bf<TX, 1, 1, ASYM>(a, scratch, sc, need, launch);
      return run_bf<TX, 2, 1, ASYM>(a, scratch, sc, need, launch);
    }
    if (a.M <= 2) return run_i8<TX, 1, false, ASYM>(a, scratch, sc, need, launch);
    if (a.M <= 4) return run_i8<TX, 2, false, ASYM>(a, scratch, sc, need, launch);
    if (a.M <= 8) return run_i8<TX, 4, false, ASYM>(a, scratch, sc, need, launch);
    return run_i8<TX, 8, false, ASYM>(a, scratch, sc, need, launch);
  }
  if (a.M <= 8) {
    if (a.group == 64) return run_bf<TX, 1, 2, ASYM>(a, scratch, sc, need, launch);
    return run_bf<TX, 1, 4, ASYM>(a, scratch, sc, need, launch);
  }
  if (a.group == 64) return run_bf<TX, 2, 2, ASYM>(a, scratch, sc, need, launch);
  return run_bf<TX, 2, 4, ASYM>(a, scratch, sc, need, launch);
}

cudaError_t run_decode_any(DType xt, const DecodeArgs& a, bool scratch, const DecodeScratch* sc,
                           DecodeNeed* need, bool launch) {
  const bool asym = a.zeros != nullptr;
  if (xt == DType::BF16)
    return asym ? run_decode<__nv_bfloat16, true>(a, scratch, sc, need, launch)
                : run_decode<__nv_bfloat16, false>(a, scratch, sc, need, launch);
  return asym ? run_decode<__half, true>(a, scratch, sc, need, launch)
              : run_decode<__half, false>(a, scratch, sc, need, launch);
}

size_t need_total_bytes(const DecodeNeed& n) {
  return n.counters * sizeof(uint32_t) + n.partials * sizeof(float) + n.records;
}

}  // namespace

cudaError_t reset_split_counters() {
  // After a bounded wait gave up, a CTA may have left an arrival counted in
  // the library's fixed array (callers' workspaces are theirs to clear).
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  float* scratch = nullptr;
  e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  return cudaMemset(reinterpret_cast<char*>(scratch) + kNoAllocPartialBytes, 0,
                    kNoAllocMaxCtas * sizeof(uint32_t));
}

size_t decode_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t decode_workspace_size(DType xt, int64_t K, int group, int64_t M, int64_t N,
                                  size_t* bytes) {
  // The need does not depend on the scheme or the epilogue.
  const DecodeArgs a{nullptr, nullptr, nullptr, nullptr, Epilogue{}, K, group, M, N, nullptr, nullptr};
  DecodeNeed n;
  const cudaError_t e = run_decode_any(xt, a, true, nullptr, &n, false);
  if (e != cudaSuccess) return e;
  *bytes = workspace_bytes(n);
  return cudaSuccess;
}

cudaError_t launch_matmul_decode(const void* x, DType xt, const uint8_t* packed,
                                 const uint16_t* scales, const uint8_t* zeros, const Epilogue& ep,
                                 int64_t K, int group, int64_t M, int64_t N, float* y,
                                 void* workspace, size_t workspace_bytes_given, cudaStream_t stream,
                                 size_t* need) {
  const DecodeArgs a{x, packed, scales, zeros, ep, K, group, M, N, y, stream};
  if (workspace == nullptr && workspace_bytes_given == 0) {
    DecodeNeed n;
    return run_decode_any(xt, a, false, nullptr, &n, true);
  }
  DecodeNeed n;
  cudaError_t e = run_decode_any(xt, a, true, nullptr, &n, false);
  if (e != cudaSuccess) return e;
  const size_t bytes = workspace_bytes(n);
  if (bytes > workspace_bytes_given || (bytes > 0 && workspace == nullptr)) {
    *need = bytes;
    return cudaErrorInvalidValue;
  }
  const DecodeScratch sc = carve_workspace(workspace, n);
  return run_decode_any(xt, a, true, &sc, &n, true);
}

cudaError_t launch_matmul_decode_noalloc(const void* x, DType xt, const uint8_t* packed,
                                         const uint16_t* scales, int64_t K, int group, int64_t M,
                                         int64_t N, float* y, cudaStream_t stream, size_t* need) {
  float* base = nullptr;
  cudaError_t e = noalloc_scratch(&base);
  if (e != cudaSuccess) return e;
  const DecodeArgs a{x, packed, scales, nullptr, Epilogue{}, K, group, M, N, y, stream};
  const DecodeScratch sc = noalloc_regions(base);
  DecodeNeed n;
  e = run_decode_any(xt, a, true, &sc, &n, true);
  if (e == cudaErrorInvalidValue && !fits(n, &sc)) *need = need_total_bytes(n);
  return e;
}

bool decode_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                      const uint8_t* packed) {
  if (xt == DType::F32) return false;
  if (M < 1 || M > 16 || N < 1) return false;
  if (K % 32 != 0 || K > (1LL << 31)) return false;
  if (!(group == 32 || group == 64 || group % 128 == 0)) return false;
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0) return false;
  if (reinterpret_cast<uintptr_t>(packed) % 16 != 0) return false;
  if (N > 0x7FFFFFFFLL) return false;
  return true;
}

}  // namespace int4lib
