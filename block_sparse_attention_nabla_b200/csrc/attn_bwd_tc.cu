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
// is needed and both orientations of a tile are equally cheap.  That lets a
// step stack ANY two kept blocks of a list into one M = 128 operand: no tile
// outside the mask is ever computed.
//
//   dkdv_tc_kernel  one unit = one key block j; a step takes the next two
//                   query blocks of j's column list (i0, i1):
//                     S  = [Q_i0; Q_i1] K_j^T     (M = 128 queries, N = 64)
//                     dP = [dO_i0; dO_i1] V_j^T
//                     P, dS per query row (one thread per row), written to
//                     shared memory as bf16
//                     dV^T += [dO_i0; dO_i1]^T P   (M = D, N = 64, K = 128)
//                     dK^T += [Q_i0; Q_i1]^T dS
//   dq_tc_kernel    one unit = one query block i; a step takes the next two
//                   key blocks of i's row list (j0, j1):
//                     S^T  = [K_j0; K_j1] Q_i^T    (M = 128 keys, N = 64)
//                     dP^T = [V_j0; V_j1] dO_i^T
//                     dS^T per key row, to shared memory as bf16
//                     dQ^T += [K_j0; K_j1]^T dS^T  (M = D, N = 64, K = 128)
//
// Every MMA has N = 64, where one issuing thread reaches about a third of the
// tensor core's rate; each kernel therefore issues its independent MMA
// streams from separate warps (S, dP, dV, dK: four issuers; S^T, dP^T, dQ^T:
// three), which together keep the tensor core fed.  One CTA per SM, persistent
// over the units.  The step's stages form a chain (load -> S, dP -> P, dS ->
// accumulate -> slot free), so every hand-off is buffered to let consecutive
// steps overlap: S and dP double-buffered in TMEM (256 columns, plus the
// accumulators), P and dS double-buffered in shared memory, and TMA rings for
// the stepped operands (dkdv: 2 stages of Q + dO; dq: 3 stages of K, and 2 of
// V, which is free as soon as dP^T completes).
//
// Warp roles (dkdv: 13 warps; dq: 12 warps):
//   warp 0       TMA producer (fixed operands per unit, stepped operands per
//                step, and the rows' 1/ln2-scaled LSE and Delta);
//   warps 1..    MMA issuers (one thread each), warp 1 also owns TMEM;
//   last eight   elementwise warps: a thread owns one row (TMEM lane) and half
//                of its 64 columns: P and dS; then the epilogue (a thread owns
//                one column d of a transposed accumulator, half of its keys or
//                queries).
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

// Shared-memory plan of dkdv_tc_kernel (byte offsets; every tile 1024-aligned).
struct DkdvSmem {
  static constexpr uint32_t k_off = 0;
  static constexpr uint32_t v_off = kFixed;
  static constexpr uint32_t kStage = 2 * kStacked + 1024;  // Q pair, dO pair, LSE2[128], Delta[128]
  static constexpr uint32_t stage0 = 2 * kFixed;
  static constexpr uint32_t p0 = stage0 + 2 * kStage;      // P[2]
  static constexpr uint32_t ds0 = p0 + 2 * kTile128;       // dS[2]
  static constexpr uint32_t bar_off = ds0 + 2 * kTile128;
  static constexpr int kBars = 17;
  static constexpr uint32_t misc_off = bar_off + kBars * 8;
  static constexpr uint32_t bytes = misc_off + 16;
  static __host__ __device__ constexpr uint32_t stage(uint32_t s) { return stage0 + s * kStage; }
  static __host__ __device__ constexpr uint32_t p(uint32_t b) { return p0 + b * kTile128; }
  static __host__ __device__ constexpr uint32_t ds(uint32_t b) { return ds0 + b * kTile128; }
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

static_assert(DkdvSmem::stage(1) % 1024 == 0 && DkdvSmem::p0 % 1024 == 0 && DkdvSmem::ds0 % 1024 == 0,
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

// P and dS of 32 columns of one row: s, dp raw accumulator words; lse2 and
// delta per column (arrays) or per row (scalars broadcast by the caller).
__device__ __forceinline__ void p_ds_pairs(const uint32_t (&sr)[32], const uint32_t (&dr)[32], float scale_log2,
                                           const float* lse2c, const float* deltac, float lse2r, float deltar,
                                           int col0, int col_lim, uint32_t* pw, uint32_t* dw) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const int c0 = 2 * c, c1 = 2 * c + 1;
    const float l0 = lse2c ? lse2c[c0] : lse2r, l1 = lse2c ? lse2c[c1] : lse2r;
    const float e0 = deltac ? deltac[c0] : deltar, e1 = deltac ? deltac[c1] : deltar;
    float p0 = ex2(fmaf(__uint_as_float(sr[c0]), scale_log2, -l0));
    float p1 = ex2(fmaf(__uint_as_float(sr[c1]), scale_log2, -l1));
    if (col0 + c0 >= col_lim) p0 = 0.f;
    if (col0 + c1 >= col_lim) p1 = 0.f;
    const float d0 = p0 * (__uint_as_float(dr[c0]) - e0), d1 = p1 * (__uint_as_float(dr[c1]) - e1);
    if (pw) pw[c] = pack_bf16x2(p0, p1);
    dw[c] = pack_bf16x2(d0, d1);
  }
}

// ============================================================== dK and dV
template <int D>
__global__ void __launch_bounds__(kDkdvThreads, 1)
    dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const float* __restrict__ lse2p, const float* __restrict__ deltap,
                   const int32_t* __restrict__ cnt_t, const int32_t* __restrict__ idx_t, int n_units, int S,
                   int nb, float scale, float scale_log2, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv, int32_t* __restrict__ status, uint64_t limit_ns) {
  static_assert(D == 128, "the tensor-core backward is built for D = 128");
  using L = DkdvSmem;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int32_t)NABLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = (uint64_t*)(smem + L::bar_off);
  uint64_t* fixed_full = bars;        // K_j, V_j landed
  uint64_t* fixed_empty = bars + 1;   // S and dP of the unit done with them
  uint64_t* in_full = bars + 2;       // [2] Q / dO pair + stats landed
  uint64_t* in_empty = bars + 4;      // [2] dV and dK of the step done with them
  uint64_t* s_full = bars + 6;        // [2] S and dP in TMEM
  uint64_t* s_free = bars + 8;        // [2] S and dP read out of TMEM
  uint64_t* pd_full = bars + 10;      // [2] P and dS written
  uint64_t* pd_empty = bars + 12;     // [2] dV and dK done with P and dS
  uint64_t* acc_full = bars + 14;
  uint64_t* acc_empty = bars + 15;
  uint64_t* drain = bars + 16;
  uint32_t* tmem_slot = (uint32_t*)(smem + L::misc_off);
  volatile int* abort_flag = (volatile int*)(smem + L::misc_off + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    mbar_init(fixed_empty, 2);
    for (int s = 0; s < 2; ++s) {
      mbar_init(in_full + s, 1);
      mbar_init(in_empty + s, 2);
      mbar_init(s_full + s, 2);
      mbar_init(s_free + s, kEwThreads);
      mbar_init(pd_full + s, kEwThreads);
      mbar_init(pd_empty + s, 2);
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

  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t g = 0, fixed_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int n = cnt_t[u];
        if (n == 0) continue;
        const int bh = u / nb, j = u - bh * nb;
        const int32_t* list = idx_t + (long long)u * nb;
        int nx0 = list[0], nx1 = n > 1 ? list[1] : nx0;  // the next step's pair, read one step early
        if (fixed_it > 0 && !(ok = mbar_wait(fixed_empty, (fixed_it - 1) & 1, abort_flag, limit_ns))) break;
        mbar_expect_tx(fixed_full, 2 * kFixed);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(smem + L::k_off + h * kTile64, &tm_k, fixed_full, h * 64, j * 64, bh);
          tma_load_3d(smem + L::v_off + h * kTile64, &tm_v, fixed_full, h * 64, j * 64, bh);
        }
        ++fixed_it;
        for (int t = 0; 2 * t < n; ++t, ++g) {
          const int i0 = nx0, i1 = nx1;
          if (2 * t + 2 < n) {
            nx0 = list[2 * t + 2];
            nx1 = 2 * t + 3 < n ? list[2 * t + 3] : nx0;
          }
          const uint32_t s = g & 1, use = g >> 1;
          if (use > 0 && !(ok = mbar_wait(in_empty + s, (use - 1) & 1, abort_flag, limit_ns))) break;
          uint8_t* st = smem + L::stage(s);
          mbar_expect_tx(in_full + s, 2 * kStacked + 1024);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(st + h * kTile128, &tm_q, in_full + s, h * 64, i0 * 64, bh);
            tma_load_3d(st + h * kTile128 + kTile64, &tm_q, in_full + s, h * 64, i1 * 64, bh);
            tma_load_3d(st + kStacked + h * kTile128, &tm_do, in_full + s, h * 64, i0 * 64, bh);
            tma_load_3d(st + kStacked + h * kTile128 + kTile64, &tm_do, in_full + s, h * 64, i1 * 64, bh);
          }
          const long long r0 = ((long long)bh * nb + i0) * 64, r1 = ((long long)bh * nb + i1) * 64;
          bulk_load(st + 2 * kStacked, lse2p + r0, 256, in_full + s);
          bulk_load(st + 2 * kStacked + 256, lse2p + r1, 256, in_full + s);
          bulk_load(st + 2 * kStacked + 512, deltap + r0, 256, in_full + s);
          bulk_load(st + 2 * kStacked + 768, deltap + r1, 256, in_full + s);
        }
      }
      // Let every copy issued land before the CTA exits.
      if (fixed_it > 0) mbar_wait(fixed_full, (fixed_it - 1) & 1, nullptr, kDrainLimitNs);
      for (uint32_t i = (g > 2 ? g - 2 : 0); i < g; ++i)
        mbar_wait(in_full + (i & 1), (i >> 1) & 1, nullptr, kDrainLimitNs);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------- S and dP issuers (one each)
    if (lane == 0) {
      const bool is_s = warp == 1;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t fixed_base = sbase + (is_s ? L::k_off : L::v_off);
      const uint32_t col = is_s ? 0u : 64u;
      uint32_t g = 0, fixed_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int n = cnt_t[u];
        if (n == 0) continue;
        if (!(ok = mbar_wait(fixed_full, fixed_it & 1, abort_flag, limit_ns))) break;
        ++fixed_it;
        const int steps = (n + 1) >> 1;
        for (int t = 0; t < steps; ++t, ++g) {
          const uint32_t s = g & 1;
          if (!(ok = mbar_wait(in_full + s, (g >> 1) & 1, abort_flag, limit_ns))) break;
          if (g >= 2 && !(ok = mbar_wait(s_free + s, ((g >> 1) - 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          const uint32_t a_base = sbase + L::stage(s) + (is_s ? 0u : kStacked);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + s * 128 + col, kmajor_desc(a_base, kTile128, kk), kmajor_desc(fixed_base, kTile64, kk),
                   idesc, kk > 0 ? 1u : 0u);
          mma_commit(s_full + s);
        }
        if (ok) mma_commit(fixed_empty);
      }
      mma_commit(drain);
    }
  } else if (warp == 3 || warp == 4) {
    // ---------------------------------------- dV and dK issuers (one each)
    if (lane == 0) {
      const bool is_v = warp == 3;
      constexpr uint32_t idesc = idesc_bf16_f32(128, 64, 1, 1);
      const uint32_t acc = tmem + kAccCol0 + (is_v ? 0u : 64u);
      uint32_t g = 0, u_local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
        const int steps = (cnt_t[u] + 1) >> 1;
        // The epilogue of the previous unit must have read the accumulators
        // (and seen its acc_full phase) before this unit overwrites or signals.
        if (u_local > 0 && !(ok = mbar_wait(acc_empty, (u_local - 1) & 1, abort_flag, limit_ns))) break;
        for (int t = 0; t < steps; ++t, ++g) {
          const uint32_t pb = g & 1;
          if (!(ok = mbar_wait(pd_full + pb, (g >> 1) & 1, abort_flag, limit_ns))) break;
          tc_fence_after();
          // A = the stacked dO (for dV) or Q (for dK) tile read MN-major: M = D
          // in two 64-column atoms, K = the 128 stacked query rows.
          const uint32_t a_base = sbase + L::stage(g & 1) + (is_v ? kStacked : 0u);
          const uint32_t b_base = sbase + (is_v ? L::p(pb) : L::ds(pb));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(acc, mnmajor_desc(a_base, kTile128, kk), mnmajor_desc(b_base, kTile128, kk), idesc,
                   (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pd_empty + pb);
          mma_commit(in_empty + (g & 1));
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      mma_commit(drain);
    }
  } else {
    // ------------------------------------- elementwise (P, dS) + epilogue
    const int half = (warp - 5) >> 2;   // which 32 of the 64 columns
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: query row of S / dP; column d of dV^T / dK^T
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t g = 0, u_local = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++u_local) {
      const int n = cnt_t[u];
      const int bh = u / nb, j = u - bh * nb;
      const int kv_lim = j == nb - 1 ? S - j * 64 : 64;
      const int steps = (n + 1) >> 1;
      for (int t = 0; t < steps; ++t, ++g) {
        const uint32_t s = g & 1;
        const bool w1 = mbar_wait(s_full + s, (g >> 1) & 1, abort_flag, limit_ns);
        const bool w2 = w1 && mbar_wait(in_full + s, (g >> 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + s * 128 + half * 32, sr);
        tmem_ld32(lane_base + s * 128 + 64 + half * 32, dr);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free + s);  // the S / dP buffer may be overwritten now
        const float* st = (const float*)(smem + L::stage(s) + 2 * kStacked);
        const float lse2 = st[r], delta = st[128 + r];
        const bool row_ok = r < 64 || 2 * t + 1 < n;
        uint32_t pw[16], dw[16];
        p_ds_pairs(sr, dr, scale_log2, nullptr, nullptr, lse2, delta, half * 32, row_ok ? kv_lim : 0, pw, dw);
        // P / dS of two steps back must have been consumed.
        const bool w3 = g < 2 || mbar_wait(pd_empty + s, ((g >> 1) - 1) & 1, abort_flag, limit_ns);
        if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
        store_half_row_sw128(smem + L::p(s), r, half, pw);
        store_half_row_sw128(smem + L::ds(s), r, half, dw);
        fence_proxy_async_smem();
        mbar_arrive(pd_full + s);
      }
      if (!ok) break;
      // epilogue: thread r owns column d = r of dV^T (half 0) or dK^T (half 1)
      const bool w4 = mbar_wait(acc_full, u_local & 1, abort_flag, limit_ns);
      if (!__all_sync(0xffffffffu, w4)) { ok = false; break; }
      tc_fence_after();
      const long long row0 = (long long)bh * S + (long long)j * 64;
      __nv_bfloat16* out = half == 0 ? dv : dk;
      const float mul = half == 0 ? 1.f : scale;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[32];
        if (steps > 0) {
          tmem_ld32(lane_base + kAccCol0 + half * 64 + h * 32, a);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) a[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (h * 32 + c < kv_lim)
            out[(row0 + h * 32 + c) * D + r] = __float2bfloat16_rn(__uint_as_float(a[c]) * mul);
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
        p_ds_pairs(sr, dr, scale_log2, lse2c, deltac, 0.f, 0.f, 0, row_ok ? 32 : 0, nullptr, dw);
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
      const float2 fa = __bfloat1622float2(a), fc = __bfloat1622float2(c);
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
                               const void* dout, const float* lse, const int32_t* cnt, const int32_t* idx,
                               const int32_t* cnt_t, const int32_t* idx_t, float* lse2p, float* deltap,
                               void* dq, void* dk, void* dv, int32_t* ws_header, cudaStream_t st) {
  if (d.dtype != NABLA_BF16 || d.D != 128) return cudaErrorInvalidValue;
  const long long rows = d.BH() * d.nb * 64;
  bwd_stats_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, lse, d.S, d.nb, rows, lse2p, deltap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_bf16(&tq, q, d, 64) || !make_map_bf16(&tk, k, d, 64) || !make_map_bf16(&tv, v, d, 64) ||
      !make_map_bf16(&tdo, dout, d, 64))
    return cudaErrorInvalidValue;
  const int n_units = (int)(d.BH() * d.nb);
  const int grid = std::min(n_units, sm_count());
  const float scale = 1.0f / sqrtf(128.0f), scale_log2 = 1.4426950408889634f * scale;
  auto k1 = dkdv_tc_kernel<128>;
  e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DkdvSmem::bytes);
  if (e != cudaSuccess) return e;
  k1<<<grid, kDkdvThreads, DkdvSmem::bytes, st>>>(tq, tk, tv, tdo, lse2p, deltap, cnt_t, idx_t, n_units, d.S, d.nb,
                                          scale, scale_log2, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv,
                                          ws_header + kWsStatus, wait_limit_ns());
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
