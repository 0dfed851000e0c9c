// Block-sparse attention backward on the 5th-generation tensor cores (sm_100a).
//
// Gradient of Eq. 4 of "∇NABLA: Neighborhood Adaptive Block-Level Attention"
// (§2.2) over the kept 64 x 64 tiles, with the mask held constant (the pages
// train through the attention only, §3.1).  With s = Q K^T (unscaled),
// P = exp(s / sqrt(D) - LSE) per query row, Delta = rowsum(dO * O):
//
//     dV = P^T dO        dP = dO V^T        dS = P * (dP - Delta)
//     dK = dS^T Q / sqrt(D)                 dQ = dS K / sqrt(D)
//
// The LSE of the forward makes every tile independent, so no online softmax
// is needed and both orientations of a tile are equally cheap.  dQ stacks any
// two kept blocks of a row list into one M = 128 operand (no tile outside the
// mask is computed); dK / dV pairs neighbouring key blocks as the forward
// pairs query blocks, so that P^T and dS^T can stay in TMEM as MMA operands,
// and computes the union of the pair's columns (rows of a key block that did
// not keep a visited query block get P = dS = 0).
//
//   dkdv_tc_kernel  one unit = two key blocks (j0, j1) stacked into 128 key
//                   rows; a step takes the next query block i of the union
//                   of their two bitmask columns:
//                     S^T  = [K_j0; K_j1] Q_i^T   (M = 128 keys, N = 64)
//                     dP^T = [V_j0; V_j1] dO_i^T
//                     P^T, dS^T per key row (one thread per row and half of
//                     the columns), written back into TMEM as bf16
//                     dV += P^T dO_i, dK += dS^T Q_i   (M = 128, N = D, A from
//                     TMEM: only Q_i and dO_i come from shared memory)
//   dq_tc_kernel    one unit = one query block i; a step takes the next two
//                   key blocks of i's row list (j0, j1):
//                     S^T  = [K_j0; K_j1] Q_i^T    (M = 128 keys, N = 64)
//                     dP^T = [V_j0; V_j1] dO_i^T
//                     dS^T per key row, to shared memory as bf16
//                     dQ^T += [K_j0; K_j1]^T dS^T  (M = D, N = 64, K = 128)
//
// Each kernel issues its independent MMA streams from separate warps (S^T,
// dP^T, dV, dK: four issuers; S^T, dP^T, dQ^T: three), which together keep
// the tensor core fed at these N = 64 / 128 shapes.  One CTA per SM,
// persistent over the units.  The step's stages form a chain (load -> S, dP
// -> P, dS -> accumulate -> slot free), so every hand-off is buffered to let
// consecutive steps overlap: S and dP double-buffered in TMEM (256 columns,
// plus the accumulators), P^T / dS^T in TMEM over them (dkdv) or dS^T
// double-buffered in shared memory (dq), and TMA rings for the stepped
// operands (dkdv: 4 stages of Q_i + dO_i; dq: 3 stages of K, and 2 of V,
// which is free as soon as dP^T completes).
//
// Warp roles (dkdv: 13 warps; dq: 12 warps):
//   warp 0       TMA producer (fixed operands per unit, stepped operands per
//                step, and the rows' 1/ln2-scaled LSE and Delta; in dkdv the
//                whole warp scans the bitmask columns for the steps);
//   warps 1..    MMA issuers (one thread each), warp 1 also owns TMEM;
//   last eight   elementwise warps: a thread owns one row (TMEM lane) and half
//                of its 64 columns: P and dS; then the epilogue (dkdv: a
//                thread writes its key row of dV or of dK; dq: a thread owns
//                one column d of dQ^T and half of its queries).
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace nabla {
namespace {

using namespace sm100;

constexpr uint32_t kTmemCols = 512;
// Elementwise warps: two per TMEM lane quarter, each taking 32 of a row's 64
// columns, so every scheduler has two of them to hide latency with.
constexpr int kEwWarps = 8;
constexpr uint32_t kEwThreads = kEwWarps * 32;
constexpr int kDkdvThreads = (5 + kEwWarps) * 32;  // producer, 4 issuers, elementwise
constexpr int kDqThreads = (4 + kEwWarps) * 32;    // producer, 3 issuers, elementwise
constexpr uint32_t kAccCol0 = 256;  // first accumulator column (after the two S/dP buffers)
constexpr uint64_t kDrainLimitNs = 1000000000ull;

constexpr uint32_t kRowBytes = 128;              // one 128-byte swizzle row = 64 bf16
constexpr uint32_t kTile64 = 64 * kRowBytes;     // 64 rows x 64 columns
constexpr uint32_t kTile128 = 128 * kRowBytes;   // 128 rows x 64 columns
constexpr uint32_t kFixed = 2 * kTile64;         // 64 rows x D = 128 (two column halves)
constexpr uint32_t kStacked = 2 * kTile128;      // 128 rows x D = 128

// Shared-memory plan of dkdv_tc_kernel (byte offsets; every tile 1024-aligned):
// the unit's stacked K and V pairs (128 rows x D, the A operands of S^T and
// dP^T) and kDkdvStages stages of one query block each: Q_i, dO_i (64 rows x
// D), LSE2 and Delta of its 64 rows, and the step record (query block,
// membership flags, steps of the unit).
constexpr int kDkdvStages = 4;
struct DkdvSmem {
  static constexpr uint32_t kp_off = 0;
  static constexpr uint32_t vp_off = kStacked;
  static constexpr uint32_t kStage = 2 * kFixed + 1024;
  static constexpr uint32_t stats = 2 * kFixed;       // within a stage: LSE2[64], Delta[64]
  static constexpr uint32_t record = 2 * kFixed + 512;  // within a stage: i, flags, n
  static constexpr uint32_t stage0 = 2 * kStacked;
  static constexpr uint32_t bar_off = stage0 + kDkdvStages * kStage;
  static constexpr int kBars = 2 + 2 * kDkdvStages + 2 + 2 + 2 + 3;
  static constexpr uint32_t misc_off = bar_off + kBars * 8;
  static constexpr uint32_t bytes = misc_off + 16;
  static __host__ __device__ constexpr uint32_t stage(uint32_t s) { return stage0 + s * kStage; }
};

// Shared-memory plan of dq_tc_kernel.
struct DqSmem {
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr uint32_t q_off = 0;
  static constexpr uint32_t do_off = kFixed;
  static constexpr uint32_t st_off = 2 * kFixed;  // LSE2[64], Delta[64] of the unit's query block
  static constexpr uint32_t k0 = st_off + 1024;   // K pairs [kKStages]
  static constexpr uint32_t v0 = k0 + kKStages * kStacked;  // V pairs [kVStages]
  static constexpr uint32_t ds0 = v0 + kVStages * kStacked; // dS^T [2]
  static constexpr uint32_t bar_off = ds0 + 2 * kTile128;
  static constexpr int kBars = 23;
  static constexpr uint32_t misc_off = bar_off + kBars * 8;
  static constexpr uint32_t bytes = misc_off + 16;
  static __host__ __device__ constexpr uint32_t k(uint32_t s) { return k0 + s * kStacked; }
  static __host__ __device__ constexpr uint32_t v(uint32_t s) { return v0 + s * kStacked; }
  static __host__ __device__ constexpr uint32_t ds(uint32_t b) { return ds0 + b * kTile128; }
};

static_assert(DkdvSmem::vp_off % 1024 == 0 && DkdvSmem::stage(1) % 1024 == 0 && DkdvSmem::kStage % 1024 == 0,
              "tile alignment");
static_assert(DqSmem::k0 % 1024 == 0 && DqSmem::v0 % 1024 == 0 && DqSmem::ds0 % 1024 == 0, "tile alignment");
static_assert(DkdvSmem::bytes <= 227 * 1024 && DqSmem::bytes <= 227 * 1024, "shared memory");

// K-major operand (rows x D, two 64-column halves of `half` bytes): the
// descriptor of MMA step kk (16 columns).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, uint32_t half, int kk) {
  return desc_sw128(base + (kk >> 2) * half + (kk & 3) * 32, 16, 1024);
}
// MN-major operand stored as rows along K (128-byte rows of 64 MN elements;
// `atom` bytes between 64-element MN atoms): MMA step kk covers K rows
// [16 kk, 16 kk + 16).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, uint32_t atom, int kk) {
  return desc_sw128(base + kk * 16 * kRowBytes, atom, 1024);
}

// 32 values (bf16 pairs) = half a 128-byte swizzled row (`half` 0: columns
// 0-31, 1: columns 32-63) of an MN-major operand tile.
__device__ __forceinline__ void store_half_row_sw128(uint8_t* tile, int row, int half, const uint32_t (&w)[16]) {
  uint8_t* r = tile + row * kRowBytes;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(r + (((4 * half + c) ^ (row & 7)) << 4)) =
        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

// P and dS of 32 columns of one row: s, dp raw accumulator words; lse2c and
// deltac the 1/ln2-scaled LSE and the Delta of the 32 columns (16-byte
// aligned shared memory, read four at a time).  keep == false (a row outside
// the mask or the sequence) gives P = dS = 0 without evaluating anything.
__device__ __forceinline__ void p_ds_cols(const uint32_t (&sr)[32], const uint32_t (&dr)[32], float scale_log2,
                                          const float* lse2c, const float* deltac, bool keep, uint32_t* pw,
                                          uint32_t* dw) {
  if (!keep) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      if (pw) pw[c] = 0u;
      dw[c] = 0u;
    }
    return;
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 l4 = reinterpret_cast<const float4*>(lse2c)[q];
    const float4 e4 = reinterpret_cast<const float4*>(deltac)[q];
    const float l[4] = {l4.x, l4.y, l4.z, l4.w}, e[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c0 = 4 * q + 2 * h, c1 = c0 + 1;
      const float p0 = ex2(fmaf(__uint_as_float(sr[c0]), scale_log2, -l[2 * h]));
      const float p1 = ex2(fmaf(__uint_as_float(sr[c1]), scale_log2, -l[2 * h + 1]));
      const float d0 = p0 * (__uint_as_float(dr[c0]) - e[2 * h]);
      const float d1 = p1 * (__uint_as_float(dr[c1]) - e[2 * h + 1]);
      if (pw) pw[2 * q + h] = pack_bf16x2(p0, p1);
      dw[2 * q + h] = pack_bf16x2(d0, d1);
    }
  }
}

// ============================================================== dK and dV
// One unit = the key blocks (j0, j1) = (2 jp, 2 jp + 1) of one (b, h), stacked
// into 128 key rows; its steps are the query blocks i that kept j0 or j1 (the
// union of the two columns of the bitmask, ascending), one per step:
//   S^T  = [K_j0; K_j1] Q_i^T     dP^T = [V_j0; V_j1] dO_i^T   (M = 128, N = 64)
//   P^T, dS^T per key row, written back into TMEM (bf16) over S^T and dP^T
//   dV  += P^T dO_i                dK  += dS^T Q_i              (M = 128, N = D,
//                                                               A from TMEM)
// so shared memory serves only the step's Q_i and dO_i to the tensor core
// (plus the unit's fixed K and V pairs).  Rows of a key block that query block
// i did not keep get P = dS = 0.
// TMEM: [0, 128) S^T / dP^T buffer 0, [128, 256) buffer 1 (S^T in the first 64
// columns, dP^T in the next 64; the bf16 P^T and dS^T of the 32 query columns
// an elementwise warp owns go into the first 16 of its own 32 columns), then
// dV [256, 384) and dK [384, 512).
template <int D>
__global__ void __launch_bounds__(kDkdvThreads, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const float* __restrict__ lse2p, const float* __restrict__ deltap,
                   const uint32_t* __restrict__ bits, const int32_t* __restrict__ cnt_t, int n_units,
                   int npairs, int S, int nb, int W, float scale, float scale_log2, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv, int32_t* __restrict__ status, uint64_t limit_ns) {
  static_assert(D == 128, "the tensor-core backward is built for D = 128");
  using L = DkdvSmem;
  constexpr int KS = kDkdvStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  uint64_t* fixed_full = bars;             // K and V pairs landed
  uint64_t* fixed_empty = bars + 1;        // S^T and dP^T of the unit done with them
  uint64_t* in_full = bars + 2;            // [KS] Q_i, dO_i, stats, record landed
  uint64_t* in_empty = bars + 2 + KS;      // [KS] dV and dK of the step done with them
  uint64_t* s_full = bars + 2 + 2 * KS;    // [2] S^T and dP^T in TMEM
  uint64_t* pd_full = s_full + 2;          // [2] P^T and dS^T written to TMEM
  uint64_t* pd_empty = s_full + 4;         // [2] dV and dK done with P^T and dS^T
  uint64_t* acc_full = s_full + 6;
  uint64_t* acc_empty = s_full + 7;
  uint64_t* drain = s_full + 8;
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    mbar_init(fixed_empty, 2);
    for (int s = 0; s < KS; ++s) {
      mbar_init(in_full + s, 1);
      mbar_init(in_empty + s, 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 2);
      mbar_init(pd_full + b, kEwThreads);
      mbar_init(pd_empty + b, 2);
    }
    mbar_init(acc_full, 2);
    mbar_init(acc_empty, kEwThreads);
    mbar_init(drain, 4);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  // A unit without steps (neither key block kept by any query block) is
  // skipped by the producer and the S^T / dP^T issuers; the dV / dK issuers and
  // the epilogue still run it (zeros).  Every role decides it the same way.
  auto unit_empty = [&](int bh, int j0) -> bool {
    const int32_t* c = cnt_t + (long long)bh * nb;
    return c[j0] + (j0 + 1 < nb ? c[j0 + 1] : 0) == 0;
  };
  auto record = [&](uint32_t s) -> const int* { return (const int*)(smem + L::stage(s) + L::record); };

  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    // The whole warp scans the unit's two bitmask columns (j0 is even, so
    // both bits sit in one word of every row), 32 query blocks per ballot;
    // lane 0 issues the copies.
    uint32_t g = 0, fixed_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int bh = u / npairs, j0 = 2 * (u - bh * npairs);
      if (unit_empty(bh, j0)) continue;
      const bool has1 = j0 + 1 < nb;
      const int j1 = has1 ? j0 + 1 : j0;  // a lone last block is loaded twice; its rows are masked
      const uint32_t fmask = has1 ? 3u : 1u;
      const uint32_t* col = bits + (long long)bh * nb * W + (j0 >> 5);
      const int sh = j0 & 31;
      auto flags_of = [&](int i) -> uint32_t { return i < nb ? (col[(long long)i * W] >> sh) & fmask : 0u; };
      int n = 0;
      for (int i0 = 0; i0 < nb; i0 += 32) n += __popc(__ballot_sync(0xffffffffu, flags_of(i0 + lane) != 0u));
      if (lane == 0) {
        if (fixed_it > 0) ok = mbar_wait(fixed_empty, (fixed_it - 1) & 1, abort_flag, limit_ns);
        if (ok) {
          mbar_expect_tx(fixed_full, 2 * kStacked);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(smem + L::kp_off + h * kTile128, &tm_k, fixed_full, h * 64, j0 * 64, bh);
            tma_load_3d(smem + L::kp_off + h * kTile128 + kTile64, &tm_k, fixed_full, h * 64, j1 * 64, bh);
            tma_load_3d(smem + L::vp_off + h * kTile128, &tm_v, fixed_full, h * 64, j0 * 64, bh);
            tma_load_3d(smem + L::vp_off + h * kTile128 + kTile64, &tm_v, fixed_full, h * 64, j1 * 64, bh);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++fixed_it;
      for (int i0 = 0; i0 < nb && ok; i0 += 32) {
        const uint32_t f = flags_of(i0 + lane);
        uint32_t m = __ballot_sync(0xffffffffu, f != 0u);
        while (m != 0u && ok) {
          const int l = __ffs(m) - 1;
          m &= m - 1u;
          const int i = i0 + l;
          const int fl = __shfl_sync(0xffffffffu, (int)f, l);
          if (lane == 0) {
            const uint32_t s = g % KS, use = g / KS;
            if (use > 0) ok = mbar_wait(in_empty + s, (use - 1) & 1, abort_flag, limit_ns);
            if (ok) {
              uint8_t* st = smem + L::stage(s);
              int* rec = (int*)(st + L::record);
              rec[0] = i;
              rec[1] = fl;
              rec[2] = n;
              mbar_expect_tx(in_full + s, 2 * kFixed + 512);  // also releases the record
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                tma_load_3d(st + h * kTile64, &tm_q, in_full + s, h * 64, i * 64, bh);
                tma_load_3d(st + kFixed + h * kTile64, &tm_do, in_full + s, h * 64, i * 64, bh);
              }
              const long long r0 = ((long long)bh * nb + i) * 64;
              bulk_load(st + L::stats, lse2p + r0, 256, in_full + s);
              bulk_load(st + L::stats + 256, deltap + r0, 256, in_full + s);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++g;
        }
      }
    }
    // Let every copy issued land before the CTA exits.
    if (lane == 0) {
      if (fixed_it > 0) mbar_wait(fixed_full, (fixed_it - 1) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (g > (uint32_t)KS ? g - KS : 0); i < g; ++i)
        mbar_wait(in_full + i % KS, (i / KS) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------- S^T and dP^T issuers (one each)
    if (lane == 0) {
      const bool is_s = warp == 1;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t a_base = sbase + (is_s ? L::kp_off : L::vp_off);
      const uint32_t col = is_s ? 0u : 64u;
      uint32_t g = 0, fixed_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int bh = u / npairs, j0 = 2 * (u - bh * npairs);
        if (unit_empty(bh, j0)) continue;
        if (!(ok = mbar_wait(fixed_full, fixed_it & 1, abort_flag, limit_ns))) break;
        ++fixed_it;
        int n = -1;  // read from the first step's record
        for (int t = 0; n < 0 || t < n; ++t, ++g) {
          const uint32_t s = g % KS, b = g & 1;
          if (!(ok = mbar_wait(in_full + s, (g / KS) & 1, abort_flag, limit_ns))) break;
          if (n < 0) n = record(s)[2];
          // buffer b is free once dV and dK of step g - 2 have read P^T / dS^T
          if (g >= 2 && !(ok = mbar_wait(pd_empty + b, ((g >> 1) - 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t b_base = sbase + L::stage(s) + (is_s ? 0u : kFixed);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + b * 128 + col, kmajor_desc(a_base, kTile128, kk), kmajor_desc(b_base, kTile64, kk), idesc,
                   kk > 0 ? 1u : 0u);
          mma_commit(s_full + b);
        }
        if (!ok) break;
        mma_commit(fixed_empty);
      }
      mma_commit(drain);
    }
  } else if (warp == 3 || warp == 4) {
    // ---------------------------------------- dV and dK issuers (one each)
    if (lane == 0) {
      const bool is_v = warp == 3;
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t acc = tmem + kAccCol0 + (is_v ? 0u : 128u);
      const uint32_t src = is_v ? 0u : 64u;  // P^T lives over S^T, dS^T over dP^T
      uint32_t g = 0, u_local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
        const int bh = u / npairs, j0 = 2 * (u - bh * npairs);
        // The epilogue of the previous unit must have read the accumulators
        // (and seen its acc_full phase) before this unit overwrites or signals.
        if (u_local > 0 && !(ok = mbar_wait(acc_empty, (u_local - 1) & 1, abort_flag, limit_ns))) break;
        int n = unit_empty(bh, j0) ? 0 : -1;
        for (int t = 0; n < 0 || t < n; ++t, ++g) {
          const uint32_t s = g % KS, b = g & 1;
          if (!(ok = mbar_wait(pd_full + b, (g >> 1) & 1, abort_flag, limit_ns))) break;
          if (n < 0) n = record(s)[2];
          tc_fence_after();
          // B = dO_i (for dV) or Q_i (for dK), MN-major: K = the 64 query
          // rows, N = D in two 64-column atoms.  A = the 16 packed columns of
          // each elementwise half: query steps kk = 0, 1 in the first half's,
          // 2, 3 in the second's.
          const uint32_t b_base = sbase + L::stage(s) + (is_v ? kFixed : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(acc, tmem + b * 128 + src + (kk >> 1) * 32 + (kk & 1) * 8,
                   desc_sw128(b_base + kk * 16 * kRowBytes, kTile64, 1024), idesc, (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pd_empty + b);
          mma_commit(in_empty + s);
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      mma_commit(drain);
    }
  } else {
    // -------------------------------- elementwise (P^T, dS^T) + epilogue
    const int half = (warp - 5) >> 2;   // which 32 of the 64 query columns
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = key row of the pair
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool upper = r >= 64;         // key block j1 (else j0); warp-uniform
    uint32_t g = 0, u_local = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
      const int bh = u / npairs, j0 = 2 * (u - bh * npairs);
      const int j = j0 + (upper ? 1 : 0);
      const bool row_ok = j < nb && j * 64 + (r & 63) < S;
      const int my_flag = upper ? 2 : 1;
      int n = unit_empty(bh, j0) ? 0 : -1;
      for (int t = 0; n < 0 || t < n; ++t, ++g) {
        const uint32_t s = g % KS, b = g & 1;
        const bool w1 = mbar_wait(s_full + b, (g >> 1) & 1, abort_flag, limit_ns);
        const bool w2 = w1 && mbar_wait(in_full + s, (g / KS) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
        tc_fence_after();
        const int* rec = record(s);
        const int fl = rec[1];
        if (n < 0) n = rec[2];
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + b * 128 + half * 32, sr);
        tmem_ld32(lane_base + b * 128 + 64 + half * 32, dr);
        tmem_ld_wait();
        const float* stc = (const float*)(smem + L::stage(s) + L::stats) + half * 32;
        const bool mine = row_ok && (fl & my_flag) != 0;
        uint32_t pw[16], dw[16];
        p_ds_cols(sr, dr, scale_log2, stc, stc + 64, mine, pw, dw);
        // into this warp's own S^T / dP^T columns, which it has read
        tmem_st16(lane_base + b * 128 + half * 32, pw);
        tmem_st16(lane_base + b * 128 + 64 + half * 32, dw);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(pd_full + b);
      }
      if (!ok) break;
      // epilogue: thread r owns key row r of the pair; half 0 writes its dV
      // row, half 1 its dK row (times 1 / sqrt(D))
      const bool w4 = mbar_wait(acc_full, u_local & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w4)) { ok = false; break; }
      tc_fence_after();
      __nv_bfloat16* out = half == 0 ? dv : dk;
      const float mul = half == 0 ? 1.f : scale;
      const long long orow = (long long)bh * S + (long long)j * 64 + (r & 63);
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t a[32];
        if (n > 0) {
          tmem_ld32(lane_base + kAccCol0 + half * 128 + c0, a);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) a[c] = 0u;
        }
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * D + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 8 * v4 + 2 * e;
              w[e] = pack_bf16x2(__uint_as_float(a[c]) * mul, __uint_as_float(a[c + 1]) * mul);
            }
            dst[v4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, kDrainLimitNs);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

// ====================================================================== dQ
template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const float* __restrict__ lse2p, const float* __restrict__ deltap,
                 const int32_t* __restrict__ cnt, const int32_t* __restrict__ idx, int n_units, int S, int nb,
                 float scale, float scale_log2, __nv_bfloat16* __restrict__ dq, int32_t* __restrict__ status,
                 uint64_t limit_ns) {
  static_assert(D == 128, "the tensor-core backward is built for D = 128");
  using L = DqSmem;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  uint64_t* fixed_full = bars;              // Q_i, dO_i, stats landed
  uint64_t* fixed_empty = bars + 1;         // S^T, dP^T and the elementwise threads done with them
  uint64_t* k_full = bars + 2;              // [KS]
  uint64_t* k_empty = k_full + KS;          // [KS] dQ^T done with the K pair
  uint64_t* v_full = k_empty + KS;          // [VS]
  uint64_t* v_empty = v_full + VS;          // [VS] dP^T done with the V pair
  uint64_t* s_full = v_empty + VS;          // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* pd_full = s_free + 2;           // [2] dS^T written
  uint64_t* pd_empty = pd_full + 2;         // [2] dQ^T done with dS^T
  uint64_t* acc_full = pd_empty + 2;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  static_assert(2 + 2 * KS + 2 * VS + 8 + 3 == L::kBars, "barrier count");
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    mbar_init(fixed_empty, 2 + kEwThreads);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 2);
      mbar_init(s_free + s, kEwThreads);
      mbar_init(pd_full + s, kEwThreads);
      mbar_init(pd_empty + s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEwThreads);
    mbar_init(drain, 3);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t g = 0, fixed_it = 0, gk = 0, gv = 0;  // steps begun, K and V pair loads issued
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int n = cnt[u];
        if (n == 0) continue;
        const int bh = u / nb, i = u - bh * nb;
        const int32_t* list = idx + (long long)u * nb;
        int nx0 = list[0], nx1 = n > 1 ? list[1] : nx0;
        if (fixed_it > 0 && !(ok = mbar_wait(fixed_empty, (fixed_it - 1) & 1, abort_flag, limit_ns))) break;
        mbar_expect_tx(fixed_full, 2 * kFixed + 512);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(smem + L::q_off + h * kTile64, &tm_q, fixed_full, h * 64, i * 64, bh);
          tma_load_3d(smem + L::do_off + h * kTile64, &tm_do, fixed_full, h * 64, i * 64, bh);
        }
        bulk_load(smem + L::st_off, lse2p + (long long)u * 64, 256, fixed_full);
        bulk_load(smem + L::st_off + 256, deltap + (long long)u * 64, 256, fixed_full);
        ++fixed_it;
        for (int t = 0; 2 * t < n; ++t, ++g) {
          const int j0 = nx0, j1 = nx1;
          if (2 * t + 2 < n) {
            nx0 = list[2 * t + 2];
            nx1 = 2 * t + 3 < n ? list[2 * t + 3] : nx0;
          }
          const uint32_t ks = g % KS, kuse = g / KS;
          if (kuse > 0 && !(ok = mbar_wait(k_empty + ks, (kuse - 1) & 1, abort_flag, limit_ns))) break;
          uint8_t* kt = smem + L::k(ks);
          mbar_expect_tx(k_full + ks, kStacked);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(kt + h * kTile128, &tm_k, k_full + ks, h * 64, j0 * 64, bh);
            tma_load_3d(kt + h * kTile128 + kTile64, &tm_k, k_full + ks, h * 64, j1 * 64, bh);
          }
          ++gk;
          const uint32_t vs = g % VS, vuse = g / VS;
          if (vuse > 0 && !(ok = mbar_wait(v_empty + vs, (vuse - 1) & 1, abort_flag, limit_ns))) break;
          uint8_t* vt = smem + L::v(vs);
          mbar_expect_tx(v_full + vs, kStacked);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(vt + h * kTile128, &tm_v, v_full + vs, h * 64, j0 * 64, bh);
            tma_load_3d(vt + h * kTile128 + kTile64, &tm_v, v_full + vs, h * 64, j1 * 64, bh);
          }
          ++gv;
        }
      }
      // Let every copy issued land before the CTA exits.
      if (fixed_it > 0) mbar_wait(fixed_full, (fixed_it - 1) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (gk > KS ? gk - KS : 0); i < gk; ++i)
        mbar_wait(k_full + i % KS, (i / KS) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (gv > VS ? gv - VS : 0); i < gv; ++i)
        mbar_wait(v_full + i % VS, (i / VS) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1 || warp == 2) {
    // -------------------------------------- S^T and dP^T issuers (one each)
    if (lane == 0) {
      const bool is_s = warp == 1;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t fixed_base = sbase + (is_s ? L::q_off : L::do_off);
      const uint32_t col = is_s ? 0u : 64u;
      uint32_t g = 0, fixed_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int n = cnt[u];
        if (n == 0) continue;
        if (!(ok = mbar_wait(fixed_full, fixed_it & 1, abort_flag, limit_ns))) break;
        ++fixed_it;
        const int steps = (n + 1) >> 1;
        for (int t = 0; t < steps; ++t, ++g) {
          const uint32_t s = g & 1;
          uint32_t a_base;
          if (is_s) {
            if (!(ok = mbar_wait(k_full + g % KS, (g / KS) & 1, abort_flag, limit_ns))) break;
            a_base = sbase + L::k(g % KS);
          } else {
            if (!(ok = mbar_wait(v_full + g % VS, (g / VS) & 1, abort_flag, limit_ns))) break;
            a_base = sbase + L::v(g % VS);
          }
          if (g >= 2 && !(ok = mbar_wait(s_free + s, ((g >> 1) - 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + s * 128 + col, kmajor_desc(a_base, kTile128, kk), kmajor_desc(fixed_base, kTile64, kk),
                   idesc, kk > 0 ? 1u : 0u);
          mma_commit(s_full + s);
          if (!is_s) mma_commit(v_empty + g % VS);
        }
        if (ok) mma_commit(fixed_empty);
      }
      mma_commit(drain);
    }
  } else if (warp == 3) {
    // --------------------------------------------------------- dQ issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 1, 1);
      uint32_t g = 0, u_local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
        const int steps = (cnt[u] + 1) >> 1;
        if (u_local > 0 && !(ok = mbar_wait(acc_empty, (u_local - 1) & 1, abort_flag, limit_ns))) break;
        for (int t = 0; t < steps; ++t, ++g) {
          const uint32_t pb = g & 1;
          if (!(ok = mbar_wait(pd_full + pb, (g >> 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          // A = the stacked K tile read MN-major (M = D), B = dS^T (N = 64 queries).
          const uint32_t a_base = sbase + L::k(g % KS);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + kAccCol0, mnmajor_desc(a_base, kTile128, kk), mnmajor_desc(sbase + L::ds(pb), kTile128, kk),
                   idesc, (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pd_empty + pb);
          mma_commit(k_empty + g % KS);
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      mma_commit(drain);
    }
  } else {
    // ------------------------------------------- elementwise (dS^T) + epilogue
    const int half = (warp - 4) >> 2;   // which 32 of the 64 query columns
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: key row of S^T / dP^T; column d of dQ^T
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float* lse2c = (const float*)(smem + L::st_off) + half * 32;
    const float* deltac = lse2c + 64;
    const int tail_keys = S - (nb - 1) * 64;  // valid keys of the last key block
    uint32_t g = 0, u_local = 0, fixed_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
      const int n = cnt[u];
      const int bh = u / nb, i = u - bh * nb;
      const int steps = (n + 1) >> 1;
      // Lists are ascending, so the last key block (the only one with padded
      // keys) can only be the list's last entry.
      const bool ends_in_tail = n > 0 && idx[(long long)u * nb + n - 1] == nb - 1;
      if (steps > 0) {
        const bool w0 = mbar_wait(fixed_full, fixed_it & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w0)) { ok = false; break; }
        ++fixed_it;
      }
      for (int t = 0; t < steps; ++t, ++g) {
        const uint32_t s = g & 1;
        const bool w1 = mbar_wait(s_full + s, (g >> 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + s * 128 + half * 32, sr);
        tmem_ld32(lane_base + s * 128 + 64 + half * 32, dr);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free + s);
        const int pos = 2 * t + (r >= 64 ? 1 : 0);  // list position of this row's key block
        const bool row_ok = pos < n && !(ends_in_tail && pos == n - 1 && (r & 63) >= tail_keys);
        uint32_t dw[16];
        p_ds_cols(sr, dr, scale_log2, lse2c, deltac, row_ok, nullptr, dw);
        const bool w3 = g < 2 || mbar_wait(pd_empty + s, ((g >> 1) - 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
        store_half_row_sw128(smem + L::ds(s), r, half, dw);
        fence_proxy_async_smem();
        mbar_arrive(pd_full + s);
      }
      if (!ok) break;
      if (steps > 0) mbar_arrive(fixed_empty);  // done with this unit's LSE2 / Delta
      // epilogue: thread r owns column d = r of dQ^T, query columns [32 half, 32 half + 32)
      const bool w4 = mbar_wait(acc_full, u_local & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w4)) { ok = false; break; }
      tc_fence_after();
      const long long row0 = (long long)bh * S + (long long)i * 64 + half * 32;
      const int q_lim = (i == nb - 1 ? S - i * 64 : 64) - half * 32;
      uint32_t a[32];
      if (steps > 0) {
        tmem_ld32(lane_base + kAccCol0 + half * 32, a);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) a[c] = 0u;
      }
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c < q_lim) dq[(row0 + c) * D + r] = __float2bfloat16_rn(__uint_as_float(a[c]) * scale);
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, kDrainLimitNs);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicCAS(status, 0, (int32_t)NABLA_ERR_TIMEOUT);
}

// ========================================================== per-row stats
// For every query row of the block-padded sequence (nb * 64 rows per (b, h)):
// LSE2 = LSE / ln 2 and Delta = sum_d dO * O (fp32) for rows < S; LSE2 = +inf
// and Delta = 0 for the padding, so padded rows get P = 0.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_stats_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ o_res,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        const float* __restrict__ lse, int S, int nb,
                                                        long long rows, float* __restrict__ lse2p,
                                                        float* __restrict__ deltap) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const long long per = (long long)nb * 64;
  const long long bh = row / per;
  const int q = (int)(row - bh * per);
  float acc = 0.f;
  if (q < S) {
    const long long base = (bh * S + q) * D;
    constexpr int E = D / 32;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + base + lane * E + e);
      const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(dout + base + lane * E + e);
      float2 fa = __bfloat1622float2(a);
      const float2 fc = __bfloat1622float2(c);
      if (o_res) {
        // O + its rounding residual: the forward's fp32 O to about 2^-16
        const float2 fr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o_res + base + lane * E + e));
        fa.x += fr.x;
        fa.y += fr.y;
      }
      acc = fmaf(fa.x, fc.x, acc);
      acc = fmaf(fa.y, fc.y, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  }
  if (lane == 0) {
    lse2p[row] = q < S ? lse[bh * S + q] * 1.4426950408889634f : INFINITY;
    deltap[row] = acc;
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const Dims& d, const void* q, const void* k, const void* v, const void* o,
                               const void* o_res, const void* dout, const float* lse, const uint32_t* bits, const int32_t* cnt,
                               const int32_t* idx, const int32_t* cnt_t, float* lse2p, float* deltap, void* dq,
                               void* dk, void* dv, int32_t* ws_header, cudaStream_t st) {
  if (d.dtype != NABLA_BF16 || d.D != 128) return cudaErrorInvalidValue;
  const long long rows = d.BH() * d.nb * 64;
  bwd_stats_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      (const __nv_bfloat16*)o, (const __nv_bfloat16*)o_res, (const __nv_bfloat16*)dout, lse, d.S, d.nb, rows,
      lse2p, deltap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_bf16(&tq, q, d, 64) || !make_map_bf16(&tk, k, d, 64) || !make_map_bf16(&tv, v, d, 64) ||
      !make_map_bf16(&tdo, dout, d, 64))
    return cudaErrorInvalidValue;
  const int n_units = (int)(d.BH() * d.nb);
  const int n_pairs = (int)(d.BH() * d.npairs);
  const int grid = std::min(n_units, sm_count());
  const float scale = 1.0f / sqrtf(128.0f), scale_log2 = 1.4426950408889634f * scale;
  auto k1 = dkdv_tc_kernel<128>;
  e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DkdvSmem::bytes);
  if (e != cudaSuccess) return e;
  k1<<<std::min(n_pairs, sm_count()), kDkdvThreads, DkdvSmem::bytes, st>>>(
      tq, tk, tv, tdo, lse2p, deltap, bits, cnt_t, n_pairs, d.npairs, d.S, d.nb, d.W, scale, scale_log2,
      (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, ws_header + kWsStatus, wait_limit_ns());
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto k2 = dq_tc_kernel<128>;
  e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DqSmem::bytes);
  if (e != cudaSuccess) return e;
  k2<<<grid, kDqThreads, DqSmem::bytes, st>>>(tq, tk, tv, tdo, lse2p, deltap, cnt, idx, n_units, d.S, d.nb, scale,
                                        scale_log2, (__nv_bfloat16*)dq, ws_header + kWsStatus, wait_limit_ns());
  return cudaGetLastError();
}

}  // namespace nabla
