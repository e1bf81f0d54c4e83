// Tensor-core dequantizing matmul for large M (prefill), sm_100a.
//
// y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] * q[n, k]): int4_matmul of
// the page "Implement INT4 group quantization, nibble packing and a
// dequantizing matmul" (problem statement), computed one K group at a time
// with the group's scale applied to each output before the fp32 running sum.
//
// A persistent CTA per SM walks output tiles of 128 weight rows (n) x 256
// activation rows (m), computed with tcgen05 MMAs (kind::f16, fp32
// accumulation in tensor memory):
//   warp 0      TMA producer: per 64-wide K stage, x [256 rows x 64] (128-byte
//               swizzle, the MMA's B operand) and the packed weights
//               [128 rows x 32 bytes], into a 4-stage shared-memory ring
//   warps 4-7   dequantizers: thread t expands weight row t of the stage from
//               nibbles to bf16/fp16 (exact: 128 + u or 1024 + u minus 136 or
//               1032, or minus 128 + z for the asymmetric scheme's unsigned
//               codes) into row t of the stage's K-major A tile (128-byte
//               swizzle) in shared memory
//   warp 1      MMA issuer: D_g = A_g * X_g^T, 16 k per MMA, into one of two
//               TMEM accumulators (128 lanes x 256 columns), one per K group;
//               a group may span stages (group 128) or share one (group 32).
//               The whole warp runs the loop and one elected lane issues, so
//               every value the MMAs take stays warp-uniform: issued from a
//               lone lane the same loop left the tensor core idle between
//               MMAs for a fifth of the time.
//   warps 8-15  epilogue: per group, load the group's accumulator from TMEM,
//               multiply by s[n, g] (TMEM lane = weight row: one scale per
//               thread) and add into fp32 registers (packed FMAs); at the end
//               of a tile, add the bias, apply ReLU and store y.
// TMEM: the two accumulators fill its 512 columns.  They let the tensor core
// run group g + 1 (or the next tile's first group) while the epilogue drains
// group g or stores a finished tile.
//
// The kernel runs at about two thirds of the tensor peak, and what holds it
// there is the hand-offs.  The MMA issuer spends about a third of its time
// waiting: most on the epilogue freeing an accumulator, then on the
// dequantizers and on the copies.  Shared memory, at about 190 bytes per
// 16-k step against 128 per cycle, is busy but not saturated.  Holding A in
// tensor memory instead (tcgen05.st from the dequantizers, MMAs reading A
// from TMEM, 192-row tiles to make room) cuts those bytes but measured
// slower.
//
// Tiles are visited in runs of kGroupM activation tiles, all weight tiles of
// a run before the next, so a run's x tiles stay in L2 while the weight tiles
// stream past (each weight tile is read from DRAM once per run).
//
// Every wait is bounded in time: a wait that gives up sets an abort flag and
// the status word, every role leaves its loops, outstanding copies and MMAs
// are drained (again with a bound) and TMEM is freed before the CTA exits.
#include <cuda.h>

#include <cstring>
#include <mutex>
#include <numeric>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace int4lib {

namespace {

#ifndef INT4_PREFILL_STAGES
#define INT4_PREFILL_STAGES 4
#endif
constexpr int kBN = 128;      // weight rows per tile (MMA M, TMEM lanes)
// Activation rows per tile (MMA N), a template parameter BM of the kernel:
// 256, or 128 for problems whose 256-row tiles would leave most SMs idle.
constexpr int kKS = 64;       // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kStages = INT4_PREFILL_STAGES;    // shared-memory ring (x and packed bytes)
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 250000000ull;  // 250 ms: far above any legitimate wait
#ifndef INT4_PREFILL_GROUP_M
#define INT4_PREFILL_GROUP_M 8
#endif
constexpr int kGroupM = INT4_PREFILL_GROUP_M;  // activation tiles per raster run
#ifndef INT4_PREFILL_PERSISTENT
#define INT4_PREFILL_PERSISTENT 1  // 1: one CTA per SM walks the tiles; 0: one CTA per tile
#endif

struct Barriers {
  uint64_t full[kStages];       // TMA bytes of stage s landed
  uint64_t empty[kStages];      // MMAs reading stage s (x) finished
  uint64_t afull[kStages];      // dequantized A of stage s written
  uint64_t tmem_full[2];        // group accumulator b complete
  uint64_t tmem_empty[2];       // epilogue finished reading accumulator b
  uint64_t drain;               // abort path: all issued MMAs finished
};

template <int BM>
struct Layout {
  static_assert(2 * BM <= static_cast<int>(kTmemCols), "two accumulators fit TMEM");
  static_assert(BM % 64 == 0, "the epilogue reads 32 columns at a time per column half");
  static constexpr int kEpiCols = BM / 2;   // accumulator columns per epilogue thread
  static constexpr int kX = BM * kKS * 2;   // 32 KB at BM = 256
  static constexpr int kP = kBN * kKS / 2;  // 4 KB
  static constexpr int kA = kBN * kKS * 2;  // 16 KB: dequantized A
  static constexpr int offX = 0;
  static constexpr int offA = offX + kStages * kX;
  static constexpr int offP = offA + kStages * kA;
  static constexpr int offBar = offP + kStages * kP;
  static constexpr int offMisc = offBar + static_cast<int>(sizeof(Barriers));
  static constexpr int kBytes = offMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};
static_assert(Layout<128>::kX % 1024 == 0 && Layout<256>::kX % 1024 == 0,
              "x stages keep the 1024-byte swizzle alignment");

// Instruction descriptor, kind::f16: D fp32, A/B bf16 (1) or fp16 (0),
// both K-major, N = BM, M = kBN.
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

// 4 packed bytes (8 consecutive k) -> 8 bf16/fp16 in natural k order, two per
// 32-bit word (the lower k in the low half): q (two's-complement nibbles), or
// q - z for unsigned codes (ASYM, zb = zero_bias(z)).
template <typename TX, bool ASYM>
__device__ __forceinline__ void expand8(uint32_t w, uint32_t zb, uint32_t* o) {
  constexpr uint32_t kx = ASYM ? Nib<TX>::kBase : Nib<TX>::kMagic;
  const uint32_t ws = w >> 4;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // byte j low nibble -> bits 0..3, byte j high nibble -> bits 16..19
    const uint32_t sel = static_cast<uint32_t>(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
    const uint32_t t = __byte_perm(w, ws, sel);
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(t), "r"(0x000F000Fu), "r"(kx));
    o[j] = Nib<TX>::sub(r, ASYM ? zb : Nib<TX>::kMagic);
  }
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

// Origin (first weight row, first activation row) of tile T in the raster.
__device__ __forceinline__ void tile_origin(int T, int num_n, int num_m, int bm, int& n0, int& m0) {
  const int per_run = kGroupM * num_n;
  const int run = T / per_run;
  const int first_m = run * kGroupM;
  const int gm = (num_m - first_m < kGroupM) ? num_m - first_m : kGroupM;
  const int r = T - run * per_run;
  n0 = (r / gm) * kBN;
  m0 = (first_m + r % gm) * bm;
}

// Work units: units u < full are whole tiles (tile u); the rest are pieces
// of the remaining (tail) tiles, ksplit per tile: unit full + v is piece
// v % ksplit of tile full + v / ksplit, and its sums go to slot v of the
// pieces' buffer.  A tile's K is cut into ksplit pieces of whole chunks of
// `spc` stages (spc * 64 k: a common multiple of the group and the stage), so
// each piece starts and ends on a group boundary; pieces of one tile are
// adjacent units.  With full = 0 every tile is split; with ksplit = 1 none.
struct Unit {
  int n0, m0;    // tile origin
  int piece;
  int slot;      // slot in the pieces' buffer, -1 for a whole tile
  int it0, it1;  // stages [it0, it1)
  int g0, g1;    // K groups [g0, g1)
};
__device__ __forceinline__ Unit unit_of(int u, int num_n, int num_m, int bm, int full, int ksplit,
                                        int nchunks, int spc, int nstages, int K, int group) {
  Unit w;
  int T, k;
  if (u < full || ksplit == 1) {
    T = u;
    w.piece = 0;
    w.slot = -1;
    k = 1;
  } else {
    const int v = u - full;
    T = full + v / ksplit;
    w.piece = v - (v / ksplit) * ksplit;
    w.slot = v;
    k = ksplit;
  }
  tile_origin(T, num_n, num_m, bm, w.n0, w.m0);
  const int c0 = w.piece * nchunks / k;
  const int c1 = (w.piece + 1) * nchunks / k;
  w.it0 = c0 * spc;
  w.it1 = c1 * spc < nstages ? c1 * spc : nstages;
  w.g0 = (w.it0 * kKS) / group;
  const int kend = w.it1 * kKS < K ? w.it1 * kKS : K;
  w.g1 = (kend + group - 1) / group;
  return w;
}

template <typename TX, bool ASYM, int BM>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_p,
    const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros, Epilogue ep,
    float* __restrict__ y, int M, int N, int K, int group, int G, int full, int ksplit, int spc,
    float* __restrict__ ypart, uint32_t* status) {
  using L = Layout<BM>;
  constexpr int kEpiCols = L::kEpiCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + L::offBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_n = (N + kBN - 1) / kBN;
  const int num_m = (M + BM - 1) / BM;
  const int num_tiles = num_n * num_m;
  const int nstages = (K + kKS - 1) / kKS;
  const int nchunks = (nstages + spc - 1) / spc;
  const int num_units = full + (num_tiles - full) * ksplit;

  const uint32_t sX = ptx::smem_u32(smem + L::offX);
  const uint32_t sA = ptx::smem_u32(smem + L::offA);
  const uint32_t sP = ptx::smem_u32(smem + L::offP);
  auto bar = [&](uint64_t* b) { return ptx::smem_u32(b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(&bars->full[s]), 1);
      ptx::mbar_init(bar(&bars->empty[s]), 1);
    }
    for (int s = 0; s < kStages; ++s) ptx::mbar_init(bar(&bars->afull[s]), 128);
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
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const WaitCtx wc{abort_flag, status};

  // Register split (per thread): 32 for the producer and MMA warps, 96 for
  // the dequantizers, 192 for the epilogue; 4*32*32 + 4*32*96 + 8*32*192 =
  // 65536, the 512 threads x 128 registers the CTA is launched with.
  if (warp < 4) {
    ptx::regs_dec<32>();
    if (warp == 0 && lane == 0) {
      // ---------------- TMA producer ----------------
      int gs = 0;  // stages issued (ring slot and phase)
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const Unit w = unit_of(u, num_n, num_m, BM, full, ksplit, nchunks, spc, nstages, K, group);
        const int n0 = w.n0, m0 = w.m0;
        for (int it = w.it0; it < w.it1; ++it, ++gs) {
          const int s = gs % kStages;
          if (!wait_bar(bar(&bars->empty[s]), ((gs / kStages) & 1) ^ 1u, wc)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bar(&bars->full[s]), L::kX + L::kP);
          ptx::tma_load_2d(sX + s * L::kX, &tm_x, it * kKS, m0, bar(&bars->full[s]));
          ptx::tma_load_2d(sP + s * L::kP, &tm_p, it * (kKS / 2), n0, bar(&bars->full[s]));
        }
      }
      if (*abort_flag) {
        // Let every issued copy land before the CTA's shared memory goes away.
        const int first = gs - kStages > 0 ? gs - kStages : 0;
        for (int j = first; j < gs; ++j) drain_bar(bar(&bars->full[j % kStages]), (j / kStages) & 1);
      }
    } else if (warp == 1) {
      // ---------------- MMA issuer ----------------
      // The whole warp waits and keeps the books; the elected lane issues the
      // MMAs and commits.  The bookkeeping between MMAs shows up directly in
      // the tensor rate, so the position inside the K group is tracked once
      // per 64-k stage when groups are whole stages (one test per four MMAs),
      // else once per 32-k half (groups of 32, 96, ...), never per MMA and
      // never by division.
      const bool leader = ptx::elect_one();
      constexpr uint32_t idesc = make_idesc<TX, BM>();
      const int span = group % kKS == 0 ? kKS : kKS / 2;  // k per bookkeeping step
      int gs = 0;
      uint32_t gc = 0;  // groups started (accumulator and phase)
      bool ok = true;
      for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
        const Unit w = unit_of(u, num_n, num_m, BM, full, ksplit, nchunks, spc, nstages, K, group);
        int gpos = 0;  // k offset of the next step inside its group (a piece starts a group)
        for (int it = w.it0; ok && it < w.it1; ++it, ++gs) {
          const int s = gs % kStages;
          const uint32_t ph = (gs / kStages) & 1;
          if (!__all_sync(0xffffffffu, wait_bar(bar(&bars->full[s]), ph, wc) &&
                                           wait_bar(bar(&bars->afull[s]), ph, wc))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t bd0 = ptx::sw128_kmajor_desc(sX + s * L::kX);
          const uint64_t ad0 = ptx::sw128_kmajor_desc(sA + s * L::kA);
          const int rem = K - it * kKS;  // k left in this tile's K (a multiple of 32)
          // One bookkeeping step: MMAs kk0 .. kk0 + nk - 1 of the stage, all in
          // one K group (K and the group are multiples of 32).
          auto step = [&](int kk0, int nk) -> bool {
            const bool first = gpos == 0;
            gpos += span;
            const bool last = gpos == group || 16 * (kk0 + nk) >= rem;
            if (gpos == group) gpos = 0;
            const uint32_t buf = gc & 1u;
            if (first) {
              if (!__all_sync(0xffffffffu,
                              wait_bar(bar(&bars->tmem_empty[buf]), ((gc >> 1) & 1u) ^ 1u, wc)))
                return false;
              ptx::tc_fence_after();
            }
            if (leader) {
              const uint32_t d = tmem_base + buf * BM;
#pragma unroll
              for (int j = 0; j < kKS / 16; ++j) {
                if (j < nk) {
                  // +32 bytes along K is +2 in a descriptor's address field.
                  const uint64_t dk = static_cast<uint64_t>(2 * (kk0 + j));
                  ptx::umma_f16(d, ad0 + dk, bd0 + dk, idesc, (first && j == 0) ? 0u : 1u);
                }
              }
              if (last) ptx::umma_commit(bar(&bars->tmem_full[buf]));
            }
            __syncwarp();
            if (last) ++gc;
            return true;
          };
          if (span == kKS) {
            ok = step(0, rem >= kKS ? kKS / 16 : rem / 16);
          } else {
            ok = step(0, 2);
            if (ok && rem > kKS / 2) ok = step(2, 2);
          }
          if (!ok) break;
          if (leader) ptx::umma_commit(bar(&bars->empty[s]));
          __syncwarp();
        }
      }
      if (*abort_flag) {
        if (leader) ptx::umma_commit(bar(&bars->drain));
        __syncwarp();
        drain_bar(bar(&bars->drain), 0);
      }
    }
  } else if (warp < 8) {
    ptx::regs_dec<96>();
    // ---------------- dequantizers: thread t owns weight row t ----------------
    const int t = threadIdx.x - 128;
    const int first_half = (t >> 2) & 1;  // rotates the two 16-byte reads to avoid bank conflicts
    int gs = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const Unit w = unit_of(u, num_n, num_m, BM, full, ksplit, nchunks, spc, nstages, K, group);
      const int n0 = w.n0;
      const uint8_t* zrow = ASYM ? zeros + static_cast<int64_t>(n0 + t < N ? n0 + t : N - 1) * G
                                 : nullptr;
      for (int it = w.it0; it < w.it1; ++it, ++gs) {
        const int s = gs % kStages;
        // The zero points of the stage's two 32-k halves (one group, or two
        // for group 32), loaded before the wait.
        uint32_t zb0 = 0u, zb1 = 0u;
        if (ASYM) {
          const int g0 = (it * kKS) / group;
          const int g1 = (it * kKS + 32) / group;
          zb0 = Nib<TX>::zero_bias(__ldg(zrow + g0));
          zb1 = Nib<TX>::zero_bias(__ldg(zrow + (g1 < G ? g1 : G - 1)));
        }
        // The stage's bytes have landed, which also means the MMAs that read
        // its A tile kStages stages ago have finished: the producer refilled
        // the stage only after they released it.
        if (!__all_sync(0xffffffffu, wait_bar(bar(&bars->full[s]), (gs / kStages) & 1, wc))) {
          ok = false;
          break;
        }
        const uint32_t prow = sP + s * L::kP + t * 32;
        const uint4 va = ptx::lds128(prow + 16 * first_half);
        const uint4 vb = ptx::lds128(prow + 16 * (first_half ^ 1));
        const uint4 lo = first_half ? vb : va;
        const uint4 hi = first_half ? va : vb;
        const uint32_t wds[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        // Row t of the K-major A tile, 128-byte swizzle: 16-byte chunk c at
        // (c ^ (t & 7)).
        const uint32_t arow = sA + s * L::kA + t * 128;
        const int swz = t & 7;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          expand8<TX, ASYM>(wds[c], c < 4 ? zb0 : zb1, o);
          ptx::sts128(arow + ((c ^ swz) << 4), make_uint4(o[0], o[1], o[2], o[3]));
        }
        ptx::fence_proxy_async_smem();  // generic-proxy writes, read by the tensor core
        ptx::mbar_arrive(bar(&bars->afull[s]));
      }
    }
  } else {
    ptx::regs_inc<192>();
    // ---------------- epilogue: lane quarter q, column half h ----------------
    const int q = warp & 3;
    const int h = (warp - 8) >> 2;
    const int row = 32 * q + lane;
    // y takes 16-byte stores when its rows are whole float4s; the pieces'
    // slots (128 x BM tile-local, rows of 128 floats) whenever the buffer is
    // 16-byte aligned.
    const bool vec_y = N % 4 == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0;
    const bool vec_p = (reinterpret_cast<uintptr_t>(ypart) & 15) == 0;
    uint32_t gc = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
      const Unit w = unit_of(u, num_n, num_m, BM, full, ksplit, nchunks, spc, nstages, K, group);
      const int n0 = w.n0, m0 = w.m0;
      const int n = n0 + row;
      float2 acc[kEpiCols / 2];
#pragma unroll
      for (int j = 0; j < kEpiCols / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
      const uint16_t* srow = scales + static_cast<int64_t>(n < N ? n : N - 1) * G;
      float s_next = w.g0 < w.g1 ? f16_bits_to_float(__ldg(srow + w.g0)) : 0.0f;
      for (int gi = w.g0; gi < w.g1; ++gi, ++gc) {
        const uint32_t buf = gc & 1u;
        const float sc = s_next;
        if (gi + 1 < w.g1) s_next = f16_bits_to_float(__ldg(srow + gi + 1));
        // Warp-uniform, as the warp-wide TMEM loads below require.
        if (!__all_sync(0xffffffffu, wait_bar(bar(&bars->tmem_full[buf]), (gc >> 1) & 1u, wc))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const float2 sc2 = make_float2(sc, sc);
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + buf * BM +
                               static_cast<uint32_t>(h * kEpiCols);
#pragma unroll
        for (int c = 0; c < kEpiCols; c += 32) {
          uint32_t r0[16], r1[16];
          ptx::tmem_ld_32x32b_x16(taddr + c, r0);
          ptx::tmem_ld_32x32b_x16(taddr + c + 16, r1);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[c / 2 + j] = __ffma2_rn(
                make_float2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1])), sc2,
                acc[c / 2 + j]);
            acc[c / 2 + 8 + j] = __ffma2_rn(
                make_float2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1])), sc2,
                acc[c / 2 + 8 + j]);
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(&bars->tmem_empty[buf]));
      }
      const int mbase = m0 + h * kEpiCols;
      // A piece of a split tile keeps its raw fp32 sums in its slot, tile-
      // local as [m - m0][n - n0] (rows of kBN floats, edges included); the
      // adding kernel sums the pieces in order, applies the epilogue and
      // writes y.
      const bool piece = w.slot >= 0;
      float* const slot = piece ? ypart + static_cast<int64_t>(w.slot) * (kBN * BM) : nullptr;
      if (ok && (piece ? vec_p : vec_y)) {
        // 16-byte stores: a 4 x 4 transpose inside each quad of lanes (two
        // butterfly steps of shuffles) leaves lane r with activation row
        // m = 4 b + r of the quad's four consecutive weight rows.  N is a
        // multiple of 4 (or the slot's rows are 128 floats), so a quad is
        // wholly inside or outside; every lane takes part in the shuffles.
        const int r = lane & 3;
        const int nq = n - r;
        const bool b1 = (r & 2) != 0, b0 = (r & 1) != 0;
#pragma unroll
        for (int b = 0; b < kEpiCols / 4; ++b) {
          float a0 = acc[2 * b].x, a1 = acc[2 * b].y, a2 = acc[2 * b + 1].x, a3 = acc[2 * b + 1].y;
          {
            const float s1 = b1 ? a0 : a2, s2 = b1 ? a1 : a3;
            const float t1 = __shfl_xor_sync(0xffffffffu, s1, 2), t2 = __shfl_xor_sync(0xffffffffu, s2, 2);
            if (b1) { a0 = t1; a1 = t2; } else { a2 = t1; a3 = t2; }
          }
          {
            const float s1 = b0 ? a0 : a1, s2 = b0 ? a2 : a3;
            const float t1 = __shfl_xor_sync(0xffffffffu, s1, 1), t2 = __shfl_xor_sync(0xffffffffu, s2, 1);
            if (b0) { a0 = t1; a2 = t2; } else { a1 = t1; a3 = t2; }
          }
          const int m = mbase + 4 * b + r;
          if (piece) {
            // Rows and columns past M and N are never read back: not stored.
            if (m < M && nq < N)
              *reinterpret_cast<float4*>(slot + (m - m0) * kBN + (nq - n0)) = make_float4(a0, a1, a2, a3);
          } else if (m < M && nq < N) {
            *reinterpret_cast<float4*>(y + static_cast<int64_t>(m) * N + nq) =
                make_float4(ep.apply(a0, nq), ep.apply(a1, nq + 1), ep.apply(a2, nq + 2), ep.apply(a3, nq + 3));
          }
        }
      } else if (ok && piece) {
        if (n < N) {
#pragma unroll
          for (int j = 0; j < kEpiCols / 2; ++j) {
            const int ml = mbase - m0 + 2 * j;
            if (m0 + ml < M) slot[ml * kBN + row] = acc[j].x;
            if (m0 + ml + 1 < M) slot[(ml + 1) * kBN + row] = acc[j].y;
          }
        }
      } else if (ok && n < N) {
#pragma unroll
        for (int j = 0; j < kEpiCols / 2; ++j) {
          const int m = mbase + 2 * j;
          if (m < M) y[static_cast<int64_t>(m) * N + n] = ep.apply(acc[j].x, n);
          if (m + 1 < M) y[static_cast<int64_t>(m + 1) * N + n] = ep.apply(acc[j].y, n);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
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

// y of the split (tail) tiles = epilogue(sum of their pieces' slots, in
// piece order).  blockIdx.y walks the tail tiles (tile full + t of the
// raster, its origin computed once per block); a thread takes four
// consecutive elements li .. li + 3 of the tile, at [m][n] = [li / kBN]
// [li % kBN] of its pieces' slots t ksplit .. t ksplit + ksplit - 1, with
// 16-byte loads (and a 16-byte store when y's rows allow).
__global__ void __launch_bounds__(256) prefill_reduce_kernel(const float* __restrict__ ypart, int ksplit,
                                                             int full, int num_n, int num_m, int bm,
                                                             int M, int N, Epilogue ep, float* __restrict__ y) {
  const int t = blockIdx.y;
  int n0, m0;
  tile_origin(full + t, num_n, num_m, bm, n0, m0);
  const int per_tile = kBN * bm;
  const int li = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (li >= per_tile) return;
  const int m = m0 + (li >> 7), n = n0 + (li & (kBN - 1));
  if (m >= M || n >= N) return;
  const float4* p = reinterpret_cast<const float4*>(ypart + static_cast<int64_t>(t) * ksplit * per_tile + li);
  float4 v = __ldcs(p);
  for (int q = 1; q < ksplit; ++q) {
    const float4 u = __ldcs(p + static_cast<int64_t>(q) * (per_tile / 4));
    v.x += u.x;
    v.y += u.y;
    v.z += u.z;
    v.w += u.w;
  }
  float* yr = y + static_cast<int64_t>(m) * N + n;
  if (n + 3 < N && N % 4 == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0) {
    *reinterpret_cast<float4*>(yr) = make_float4(ep.apply(v.x, n), ep.apply(v.y, n + 1), ep.apply(v.z, n + 2),
                                                 ep.apply(v.w, n + 3));
  } else {
    const float vv[4] = {v.x, v.y, v.z, v.w};
    for (int i = 0; i < 4 && n + i < N; ++i) yr[i] = ep.apply(vv[i], n + i);
  }
}
static_assert(kBN == 128, "the adding kernel splits a slot index by shifts");

#ifndef INT4_PREFILL_TAIL_SPLIT
#define INT4_PREFILL_TAIL_SPLIT 1  // cut the tiles of a last partial wave into K pieces
#endif
#ifndef INT4_PREFILL_SMALL_BM
#define INT4_PREFILL_SMALL_BM 1  // 128-row activation tiles for problems of less than one wave
#endif

// Activation rows per tile: 128 when the 256-row tiling leaves SMs idle and
// the 128-row one still fits one wave (twice the CTAs, each with half the
// MMAs and half the stores of y, which a single CTA per SM issues at about
// 16 GB/s: 8 us for a 128 x 256 fp32 tile), else 256.
int choose_bm(int64_t M, int64_t N) {
  const int64_t sms = num_sms();
  const int64_t nt = (N + kBN - 1) / kBN;
  const int64_t t256 = nt * ((M + 255) / 256);
  const int64_t t128 = nt * ((M + 127) / 128);
  return (INT4_PREFILL_SMALL_BM && t256 < sms && t128 <= sms) ? 128 : 256;
}

// How to cut the work: whole tiles, except that the tiles of a last,
// partial wave (all of them when there are fewer tiles than SMs) may be cut
// into ksplit K pieces, so that the pieces fill that wave.  Pieces write and
// re-read their fp32 sums and need the adding kernel.  The estimate
// (calibrated on B200): a unit costs its share of the tile's stages at about
// 0.6 us per 64-k stage of a 128 x 256 tile (half that at 128 rows), about
// 3 us to start and finish, and its store of a tile of fp32 sums at about
// 16 GB/s per SM; whole waves come first, then one wave of the tail's
// units, then the pieces' round trip through HBM and about 1 us for the
// adding kernel.
struct SplitPlan {
  int ksplit = 1;
  int full = 0;   // leading whole-tile units
  int ntail = 0;  // tiles cut into pieces
  int spc = 1;    // stages per chunk: a common multiple of the group and the 64-k stage
};
SplitPlan plan_split(int64_t K, int group, int64_t M, int64_t N, int bm) {
  SplitPlan p;
  const int64_t g64 = std::gcd(static_cast<int64_t>(group), static_cast<int64_t>(kKS));
  p.spc = static_cast<int>(group / g64);  // lcm(group, 64) / 64
  const int64_t nstages = (K + kKS - 1) / kKS;
  const int64_t nchunks = (nstages + p.spc - 1) / p.spc;
  const int64_t tiles = ((N + kBN - 1) / kBN) * ((M + bm - 1) / bm);
  const int64_t sms = num_sms();
  const int64_t waves = tiles / sms;
  const int64_t tail = tiles - waves * sms;
  if (tail == 0 || nchunks < 2 || !INT4_PREFILL_TAIL_SPLIT && waves > 0) return p;
  const double stage_us = 0.6 * bm / 256.0, unit_us = 3.0, reduce_us = 1.0, hbm_bytes_per_us = 6.0e6;
  const double store_us = static_cast<double>(kBN) * bm * 4 / 16.0e3;
  const double tile_us = static_cast<double>(nstages) * stage_us;
  const double whole = tile_us + unit_us + store_us;
  const double tile_bytes = static_cast<double>(kBN) * bm * 4;
  double best = whole;  // k = 1: the tail as one more wave of whole tiles
  for (int64_t k = 2; k <= 8 && k <= nchunks && tail * k <= sms; ++k) {
    const double t = tile_us / static_cast<double>(k) + unit_us + store_us +
                     static_cast<double>(tail * k) * tile_bytes * 2 / hbm_bytes_per_us + reduce_us;
    if (t < best) {
      best = t;
      p.ksplit = static_cast<int>(k);
    }
  }
  if (p.ksplit > 1) {
    p.full = static_cast<int>(waves * sms);
    p.ntail = static_cast<int>(tail);
  }
  return p;
}

size_t split_bytes(const SplitPlan& sp, int bm) {
  return sp.ksplit > 1 ? static_cast<size_t>(sp.ntail) * sp.ksplit * kBN * bm * sizeof(float) : 0;
}

template <typename TX, bool ASYM, int BM>
cudaError_t launch_typed(const TX* x, const uint8_t* packed, const uint16_t* scales,
                         const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                         int64_t N, float* y, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
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
  auto kern = prefill_kernel<TX, ASYM, BM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  // Split K only when the caller's workspace holds the pieces' sums (past
  // the counters a decode call keeps at its start).
  SplitPlan sp = plan_split(K, group, M, N, BM);
  const size_t part_bytes = split_bytes(sp, BM);
  // The pieces' buffer takes 16-byte loads and stores: a workspace too small
  // or not 16-byte aligned runs the tiles whole.
  if (sp.ksplit > 1 &&
      (workspace == nullptr || workspace_bytes < kWorkspaceCounterBytes + part_bytes ||
       (reinterpret_cast<uintptr_t>(workspace) & 15) != 0))
    sp = SplitPlan{};
  float* ypart = sp.ksplit > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                          kWorkspaceCounterBytes)
                               : nullptr;
  const int64_t num_tiles = ((N + kBN - 1) / kBN) * ((M + BM - 1) / BM);
  const int64_t units = sp.full + (num_tiles - sp.full) * sp.ksplit;
  const int64_t sms = num_sms();
  const int64_t ctas = INT4_PREFILL_PERSISTENT ? (units < sms ? units : sms) : units;
  const dim3 grid(static_cast<unsigned>(ctas));  // persistent: one CTA per SM
  const int G = static_cast<int>((K + group - 1) / group);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(tx, tp, scales, zeros, ep, y, static_cast<int>(M),
                                              static_cast<int>(N), static_cast<int>(K), group, G,
                                              sp.full, sp.ksplit, sp.spc, ypart, status);
  e = cudaGetLastError();
  if (e != cudaSuccess || ypart == nullptr) return e;
  // One thread per four elements of each tail tile.
  const int64_t bx = (static_cast<int64_t>(kBN) * BM / 4 + 255) / 256;
  prefill_reduce_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(sp.ntail)), 256, 0, stream>>>(
      ypart, sp.ksplit, sp.full, static_cast<int>((N + kBN - 1) / kBN),
      static_cast<int>((M + BM - 1) / BM), BM, static_cast<int>(M), static_cast<int>(N), ep, y);
  return cudaGetLastError();
}

template <typename TX>
cudaError_t launch_tx(const TX* x, const uint8_t* packed, const uint16_t* scales,
                      const uint8_t* zeros, const Epilogue& ep, int64_t K, int group, int64_t M,
                      int64_t N, float* y, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  const bool small = choose_bm(M, N) == 128;
  if (zeros != nullptr)
    return small ? launch_typed<TX, true, 128>(x, packed, scales, zeros, ep, K, group, M, N, y, workspace,
                                              workspace_bytes, stream)
                 : launch_typed<TX, true, 256>(x, packed, scales, zeros, ep, K, group, M, N, y, workspace,
                                              workspace_bytes, stream);
  return small ? launch_typed<TX, false, 128>(x, packed, scales, nullptr, ep, K, group, M, N, y, workspace,
                                             workspace_bytes, stream)
               : launch_typed<TX, false, 256>(x, packed, scales, nullptr, ep, K, group, M, N, y, workspace,
                                             workspace_bytes, stream);
}

}  // namespace

bool prefill_supported(DType xt, int64_t K, int group, int64_t M, int64_t N, const void* x,
                       const uint8_t* packed) {
  if (xt == DType::F32) return false;
  if (M < 1 || N < 1 || K < 1) return false;
  if (K % 32 != 0 || group % 32 != 0) return false;
  if (K > (1LL << 30) || M > (1LL << 30) || N > (1LL << 30)) return false;
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0 || reinterpret_cast<uintptr_t>(packed) % 16 != 0)
    return false;
  if (((N + kBN - 1) / kBN) * ((M + 127) / 128) > 0x7FFFFFFFLL) return false;
  return true;
}

cudaError_t launch_matmul_prefill(const void* x, DType xt, const uint8_t* packed,
                                  const uint16_t* scales, const uint8_t* zeros, const Epilogue& ep,
                                  int64_t K, int group, int64_t M, int64_t N, float* y,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (xt == DType::BF16)
    return launch_tx(static_cast<const __nv_bfloat16*>(x), packed, scales, zeros, ep, K, group, M,
                     N, y, workspace, workspace_bytes, stream);
  return launch_tx(static_cast<const __half*>(x), packed, scales, zeros, ep, K, group, M, N, y,
                   workspace, workspace_bytes, stream);
}

size_t prefill_workspace_size(int64_t K, int group, int64_t M, int64_t N) {
  const int bm = choose_bm(M, N);
  const SplitPlan sp = plan_split(K, group, M, N, bm);
  return sp.ksplit > 1 ? kWorkspaceCounterBytes + split_bytes(sp, bm) : 0;
}

}  // namespace int4lib
